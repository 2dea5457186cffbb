// fa_fwd.cuh -- forward attention kernel for sm_100a.
//
// Computes O = softmax(scale Q K^T + mask) V and LSE for one block of 256
// query rows of one (sequence, query head) per CTA, streaming K and V tiles
// of 128 rows through shared memory ("FlashAttention优化" 3.1: Q blocks stay
// on chip while K/V blocks stream past; paper review 方法 item 1: no N x N
// matrix is written back, only O).  The softmax statistics follow the online
// recurrence of "FlashAttention优化" 3.2.1 (running max m, running sum l,
// l <- e^(m_old - m_new) l + sum exp(x - m_new)) and the accumulated output
// is rescaled by the same factor (paper review 方法 item 2).
//
// B200 design (not the pages' A100 r = c = 64 design):
//  * Two 128-row Q tiles per CTA share every K/V tile (halves L2->SMEM
//    traffic) and ping-pong on the tensor core: while softmax works on
//    tile 0, the MMA warp runs tile 1's products and vice versa.
//  * S = Q K^T and O += P V run as tcgen05.mma (M = 128) with fp32
//    accumulators in TMEM: S_t at columns [128 t, 128 t + 128), O_t at
//    [256 + d t, 256 + d t + d).  Where P (bf16) lives depends on d:
//      d = 128: P overwrites the first 64 columns of S_t and feeds PV from
//               TMEM (TS MMA).  Keeping P out of shared memory matters here:
//               with P in shared memory the tensor core's operand reads, the
//               TMA fills and the P stores need ~384 KB per K/V tile, about
//               3k cycles of shared-memory bandwidth against 2k of MMA work.
//      d = 64:  P goes to its own 128B-swizzled shared-memory tile, so S_t's
//               columns are free as soon as the softmax has read them; the
//               MMA warp issues the next S_t at once and the softmax (the
//               bottleneck at d = 64, bound by MUFU exp2) never waits for PV.
//  * One TMA warp fills a ring of K/V stages (mbarrier full/empty pairs),
//    one thread issues all MMAs, and each softmax warpgroup owns one Q tile:
//    a thread owns one query row (TMEM lane), so row max and row sum are
//    in-thread reductions.
//  * Exponentials are exp2 with the scale folded in (x = s scale log2 e).
//    The running max m is kept when a tile's max exceeds it by little, which
//    saves O rescales and is exact in real arithmetic: the final O / l uses
//    the same reference.  In bf16 it is not free: P~ = 2^(x - m) may exceed 1
//    and its rounding in P V (relative 2^-9) then falls on the weight of an
//    element the row may be dominated by, scaling that row of O as a whole
//    and biasing D = rowsum(dO o O) in the backward.  So m moves when the
//    tile's max exceeds it by more than RESCALE_LOG2 (P~ stays <= 256), or
//    exceeds it at all while 2^(m_tile - m), the largest new P~, is more than
//    MOVE_SHARE times the row's running sum l: an element kept under a stale
//    max then ends with at most a ninth of its row's weight, and a dominant
//    element always gets P~ = 1 exactly.  O in TMEM is rescaled only for the
//    rows whose max moved.
//  * Causal attention skips every K/V tile above the diagonal; only the
//    last tile of each Q tile is masked element-wise.  Variable-length
//    batches mask key columns past the sequence end and never store rows
//    past it.
#pragma once
#include "fa_common.cuh"
#include "sm100.cuh"

namespace fa {

template <int D>
struct FwdLayout {
  static constexpr int TILE = 128 * D * 2;     // bytes of one 128 x D bf16 tile
  static constexpr int NS = (D == 128) ? 3 : 6;  // K/V ring stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = 2 * TILE;
  static constexpr bool P_SMEM = (D == 64);             // where P lives (see above)
  static constexpr int OFF_P = OFF_RING + NS * TILE;    // 2 x 128 x 128 bf16 if P_SMEM
  static constexpr int OFF_BAR = OFF_P + (P_SMEM ? 2 * 32768 : 0);
  // q_full[2] kv_full[NS] kv_empty[NS] s_full[2] s_free[2] p_full[2] p_free[2] drain[1]
  static constexpr int NBAR = 2 + 2 * NS + 9;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // block-sparse mode: the CTA's K/V tile list (uint16 [FA_SPARSE_MAX_TILES]),
  // which Q tile owns each K/V tile (uint32 bits [2][FA_SPARSE_MAX_TILES/32])
  // and the list's length
  static constexpr int OFF_LIST = OFF_MISC + 16;
  static constexpr int OFF_OWN = OFF_LIST + 2 * FA_SPARSE_MAX_TILES;
  static constexpr int OFF_NLIST = OFF_OWN + 2 * (FA_SPARSE_MAX_TILES / 32) * 4;
  static constexpr int BYTES = OFF_NLIST + 16;
  static constexpr int ALLOC = BYTES + 1024;   // slack for 1024-byte alignment
};

// warps 0-7: softmax (two warpgroups); warp 8: TMA; warp 9: MMA; warps 10-11
// only give their registers to the softmax warpgroups
constexpr int FWD_THREADS = 384;
constexpr int FWD_REGS_SOFTMAX = 216;   // warpgroups 0-1 after setmaxnreg.inc
constexpr int FWD_REGS_CTRL = 72;       // warpgroup 2 after setmaxnreg.dec
static_assert(128 * (2 * FWD_REGS_SOFTMAX + FWD_REGS_CTRL) <= 65536 &&
                  2 * (FWD_REGS_SOFTMAX - 168) * 128 == (168 - FWD_REGS_CTRL) * 128,
              "register split");
// When the running max moves (see the header comment): always once the tile
// max exceeds it by more than RESCALE_LOG2 (log2 units), and for any excess
// while 2^excess > MOVE_SHARE * l.  Measured on B200 against moving on every
// increase (forward TFLOP/s): the rule moves the max on 0.5-1.6% of
// (row, tile) steps instead of 14-27% in a CPU model of the kernel, with the
// same dK and dV errors on the workloads whose rows are dominated by one key.
constexpr float RESCALE_LOG2 = 8.0f;
constexpr float MOVE_SHARE = 0.125f;
// Pairs out of every 8 column pairs whose exp2 runs on the FMA pipe
// (ex2_poly2, packed) instead of MUFU.  Measured on B200 with the packed
// loop (forward TFLOP/s for 0 / 1 / 2 / 3 pairs of 8):
//   d = 64,  causal H=16 N=4096:   524 / 522 / 514 / 498
//   d = 64,  causal H=16 N=16384:  740 / 720 / 697 / 667
//   d = 128, GQA B=2 Hq=32 N=4096: 979 / 990 / 997 / 1001
//   d = 128, causal H=16 N=65536 (power-capped; per 100 MHz of SM clock):
//            69.9 / 72.6 / 72.4 / 71.3
// At d = 64 the softmax's latency chain, not MUFU throughput, sets the pace
// and the polynomial only lengthens it; at d = 128 the MUFU queue is shared
// by both warpgroups between longer MMA phases and a quarter of the pairs on
// the FMA pipe shortens it.
template <int D>
constexpr int exp2_poly_pairs_of_8() {
  return D == 128 ? 2 : 0;
}

template <int D, bool CAUSAL, bool SPARSE = false>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using L = FwdLayout<D>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- work item
  // The (sequence, kv head) pairs are cut into chunks of order_chunk pairs
  // (with their query heads); within a chunk the Q block index is slowest,
  // heaviest blocks first.  One chunk of every pair unless the K and V of all
  // pairs are at least twice the L2: then a chunk holds at least two waves of
  // blocks and the blocks in flight share the chunk's K/V tiles in L2 (at
  // B=1, H=16, N=65536, d=128 the K/V set is 512 MiB).
  const unsigned g = (unsigned)p.group;
  const unsigned npairs = (unsigned)(p.B * p.Hkv);
  const unsigned chunk = (unsigned)p.order_chunk;
  const unsigned per_pair = g * (unsigned)p.num_qblocks;
  const unsigned cidx = blockIdx.x / (chunk * per_pair);
  const unsigned rr = blockIdx.x - cidx * chunk * per_pair;
  const unsigned pairs = min(chunk, npairs - cidx * chunk);
  const int qb = p.num_qblocks - 1 - (int)(rr / (pairs * g));   // heaviest blocks first
  const unsigned rem = rr % (pairs * g);
  const unsigned pair = cidx * chunk + rem / g;
  const int b = (int)(pair / (unsigned)p.Hkv);
  const int h = (int)((pair % (unsigned)p.Hkv) * g + rem % g);
  int seq_start = 0, len = p.N, bcoord = b;
  if (p.cu_seqlens != nullptr) {
    seq_range(p.cu_seqlens, b, p.total, &seq_start, &len);
    bcoord = 0;
  }
  const int q0 = qb * 256;
  if (q0 >= len) return;
  const int hk = h / p.group;
  const int nkv_all = (len + 127) / 128;
  uint16_t* s_list = reinterpret_cast<uint16_t*>(smem + L::OFF_LIST);
  uint32_t* s_own = reinterpret_cast<uint32_t*>(smem + L::OFF_OWN);
  int* s_nlist = reinterpret_cast<int*>(smem + L::OFF_NLIST);
  if (SPARSE && warp == 10) {
    // Block-sparse: the K/V tiles this CTA streams are those allowed for
    // either of its two Q tiles (and on or below the diagonal when causal),
    // in increasing order; a Q tile masks the ones it does not own.
    const uint8_t* mrow = p.bmask + (long)b * p.bm_sb + (long)hk * p.bm_sh;
    int cnt = 0;
    for (int c0 = 0; c0 < nkv_all; c0 += 32) {
      const int c = c0 + lane;
      bool own[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int qt = 2 * qb + t;
        own[t] = c < nkv_all && 128 * qt < len && (!CAUSAL || c <= qt) &&
                 mrow[(long)qt * p.bm_nt + c] != 0;
      }
      const uint32_t b0 = __ballot_sync(0xffffffffu, own[0]);
      const uint32_t b1 = __ballot_sync(0xffffffffu, own[1]);
      const uint32_t any = b0 | b1;
      if (lane == 0) {
        s_own[c0 >> 5] = b0;
        s_own[FA_SPARSE_MAX_TILES / 32 + (c0 >> 5)] = b1;
      }
      if ((any >> lane) & 1u) s_list[cnt + __popc(any & ((1u << lane) - 1u))] = (uint16_t)c;
      cnt += __popc(any);
    }
    if (lane == 0) *s_nlist = cnt;
  }
  int n_t[2];
  if (!SPARSE) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int r0 = q0 + 128 * t;
      n_t[t] = (r0 >= len) ? 0 : (CAUSAL ? min(nkv_all, r0 / 128 + 1) : nkv_all);
    }
  }

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* ring = smem + L::OFF_RING;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;   // S_t in TMEM (MMA commit)
  uint64_t* s_free = s_full + 2;      // S_t read out by the softmax (128 threads)
  uint64_t* p_full = s_free + 2;      // P_t written, O_t rescaled (128 threads)
  uint64_t* p_free = p_full + 2;      // PV_t done: P_t buffer free, O_t current (commit)
  uint64_t* drain = p_free + 2;
  uint8_t* sP = smem + L::OFF_P;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, 128);
      mbar_init(p_full + i, 128);
      mbar_init(p_free + i, 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{&g_fa_error, abort_flag, p.wait_limit_ns};
  if (SPARSE) {
    // both Q tiles step through the whole list (masking the tiles they do
    // not own), so the dense issue order of the MMA warp applies unchanged
    const int nl = *s_nlist;
#pragma unroll
    for (int t = 0; t < 2; ++t) n_t[t] = (q0 + 128 * t >= len) ? 0 : nl;
  }
  const int nmax = max(n_t[0], n_t[1]);

  if (warp >= 8) {
  // ============================================================== warpgroup 2
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(FWD_REGS_CTRL));
  if (warp == 8) {
    // ============================================================ TMA producer
    if (lane == 0) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (n_t[t] == 0) continue;
        mbar_arrive_expect_tx(q_full + t, L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sQ + t * L::TILE + c * 16384, &tmQ, q_full + t, c * 64, h,
                      seq_start + q0 + 128 * t, bcoord);
      }
      int issued = 0;
      for (int n = 0; n < 2 * nmax; ++n) {
        const int stage = n % NS;
        if (!mbar_wait(kv_empty + stage, ((n / NS) & 1) ^ 1, wd, ERR_FWD_KV_EMPTY)) break;
        const CUtensorMap* map = (n & 1) ? &tmV : &tmK;
        mbar_arrive_expect_tx(kv_full + stage, L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(ring + stage * L::TILE + c * 16384, map, kv_full + stage, c * 64, hk,
                      seq_start + 128 * (SPARSE ? (int)s_list[n >> 1] : (n >> 1)), bcoord);
        issued = n + 1;
      }
      if (*abort_flag) {
        // loads still in flight must land before the CTA may exit
        for (int n = max(0, issued - NS); n < issued; ++n)
          mbar_wait_drain(kv_full + n % NS, (n / NS) & 1, p.wait_limit_ns);
        for (int t = 0; t < 2; ++t)
          if (n_t[t] > 0) mbar_wait_drain(q_full + t, 0, p.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      // descriptors built once: Q tiles, the ring (K-major view for S, N-major
      // view for V as the B operand of PV) and the P tiles (K-major)
      const SDesc dq = sdesc_make(smem_u32(sQ), 16, 1024);
      const SDesc dk = sdesc_make(smem_u32(ring), 16, 1024);
      const SDesc dv = sdesc_make(smem_u32(ring), 16384, 1024);
      const SDesc dp = sdesc_make(smem_u32(sP), 16, 1024);
      // S_t = Q_t K^T : A = Q_t (K-major), B = K tile (K-major), K-dim = d
      auto issue_s = [&](int t, int stage) {
        const uint32_t dt = tmem + t * 128;
        const uint32_t qo = t * L::TILE, ko = stage * L::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(dt, sdesc_at(dq, qo + off), sdesc_at(dk, ko + off), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // O_t (+)= P_t V : A = P_t (TMEM, or smem K-major), B = V tile (N = d
      // contiguous)
      auto issue_pv = [&](int t, int stage, bool acc) {
        const uint32_t dt = tmem + 256 + t * D;
        const uint32_t vo = stage * L::TILE;
        if constexpr (L::P_SMEM) {
          const uint32_t po = t * 32768;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(dt, sdesc_at(dp, po + (kk >> 2) * 16384 + (kk & 3) * 32),
                   sdesc_at(dv, vo + kk * 2048), idesc_o, (acc || kk > 0) ? 1u : 0u);
        } else {
          const uint32_t at = tmem + t * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(dt, at + kk * 8, sdesc_at(dv, vo + kk * 2048), idesc_o,
                   (acc || kk > 0) ? 1u : 0u);
        }
      };
      // (nmax = 0 only in block-sparse mode, for a CTA with an empty list:
      // nothing is loaded and nothing issued)
      bool ok = nmax > 0;
      for (int t = 0; t < 2 && ok; ++t)
        if (n_t[t] > 0) ok = mbar_wait(q_full + t, 0, wd, ERR_FWD_Q_FULL);
      if (ok) ok = mbar_wait(kv_full + 0, 0, wd, ERR_FWD_KV_FULL);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (n_t[t] > 0) {
            issue_s(t, 0);
            mma_commit(s_full + t);
          }
        mma_commit(kv_empty + 0);
      }
      if constexpr (L::P_SMEM) {
        // Per K/V tile j and Q tile t: S_t of tile j+1 as soon as the softmax
        // has read S_t^j, then PV_t^j once P_t^j is in shared memory.
        for (int j = 0; ok && j < nmax; ++j) {
          const int nv = 2 * j + 1, sv = nv % NS;
          const int nk = 2 * j + 2, sk = nk % NS;
          const bool has_next = j + 1 < nmax;
          if (has_next) {
            if (!(ok = mbar_wait(kv_full + sk, (nk / NS) & 1, wd, ERR_FWD_KV_FULL))) break;
            tc_fence_after();
          }
          if (!(ok = mbar_wait(kv_full + sv, (nv / NS) & 1, wd, ERR_FWD_KV_FULL))) break;
          tc_fence_after();
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (has_next && j + 1 < n_t[t]) {
              if (!(ok = mbar_wait(s_free + t, j & 1, wd, ERR_FWD_S_FREE))) break;
              tc_fence_after();
              issue_s(t, sk);
              mma_commit(s_full + t);
            }
            if (j < n_t[t]) {
              if (!(ok = mbar_wait(p_full + t, j & 1, wd, ERR_FWD_P_FULL))) break;
              tc_fence_after();
              issue_pv(t, sv, j > 0);
              mma_commit(p_free + t);
            }
          }
          if (!ok) break;
          if (has_next) mma_commit(kv_empty + sk);
          mma_commit(kv_empty + sv);
        }
      } else {
        // P aliases S_t, so S_t of tile j+1 follows PV_t^j; the two Q tiles
        // ping-pong: PV_0^j, S_0^{j+1}, PV_1^j, S_1^{j+1}.
        for (int j = 0; ok && j < nmax; ++j) {
          const int nv = 2 * j + 1, sv = nv % NS;
          const int nk = 2 * j + 2, sk = nk % NS;
          const bool has_next = j + 1 < nmax;
          if (!(ok = mbar_wait(kv_full + sv, (nv / NS) & 1, wd, ERR_FWD_KV_FULL))) break;
          tc_fence_after();
          if (j < n_t[0]) {
            if (!(ok = mbar_wait(p_full + 0, j & 1, wd, ERR_FWD_P_FULL))) break;
            tc_fence_after();
            issue_pv(0, sv, j > 0);
            mma_commit(p_free + 0);
          }
          if (has_next) {
            if (!(ok = mbar_wait(kv_full + sk, (nk / NS) & 1, wd, ERR_FWD_KV_FULL))) break;
            tc_fence_after();
            if (j + 1 < n_t[0]) {
              issue_s(0, sk);
              mma_commit(s_full + 0);
            }
          }
          if (j < n_t[1]) {
            if (!(ok = mbar_wait(p_full + 1, j & 1, wd, ERR_FWD_P_FULL))) break;
            tc_fence_after();
            issue_pv(1, sv, j > 0);
            mma_commit(p_free + 1);
          }
          mma_commit(kv_empty + sv);
          if (has_next) {
            if (j + 1 < n_t[1]) {
              issue_s(1, sk);
              mma_commit(s_full + 1);
            }
            mma_commit(kv_empty + sk);
          }
        }
      }
      // every MMA issued above completes before TMEM can be released
      if (nmax > 0) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0, p.wait_limit_ns);
      }
    }
    __syncwarp();
  }
  } else {
    // ============================================================ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(FWD_REGS_SOFTMAX));
    const int t = warp >> 2;
    const int r = (warp & 3) * 32 + lane;                 // row in tile == TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * D;
    const int qrow = q0 + 128 * t + r;
    const float c2 = p.scale_log2;
    const int n = n_t[t];
    float m = -INFINITY;   // running max of s * scale * log2(e)
    float l = 0.f;         // running sum of exp2(x - m)
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full + t, j & 1, wd, ERR_FWD_S_FULL));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tS + 0, s + 0);
      tmem_ld32(tS + 32, s + 32);
      tmem_wait_ld32(s + 0);
      tmem_wait_ld32(s + 32);
      tmem_ld32(tS + 64, s + 64);      // second half loads while the first half is scanned
      tmem_ld32(tS + 96, s + 96);
      // last tile of this Q tile: sequence end and/or causal diagonal mask;
      // block-sparse: any tile may be cut by them, and a tile this Q tile
      // does not own is masked whole
      bool masked = (j == n - 1);
      int lim;
      if constexpr (SPARSE) {
        const int kt = s_list[j];
        const bool own = (s_own[t * (FA_SPARSE_MAX_TILES / 32) + (kt >> 5)] >> (kt & 31)) & 1u;
        lim = len - 128 * kt;
        if (CAUSAL) lim = min(lim, qrow + 1 - 128 * kt);
        if (!own) lim = 0;
        masked = lim < 128;
      } else {
        lim = len - 128 * j;
        if (CAUSAL) lim = min(lim, qrow + 1 - 128 * j);
      }
      if (masked) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= lim) s[c] = 0xff800000u;   // -inf
      }
      // row max: four independent chains of 3-input max
      float mx[4] = {__uint_as_float(s[0]), __uint_as_float(s[1]), __uint_as_float(s[2]),
                     __uint_as_float(s[3])};
#pragma unroll
      for (int c = 4; c < 64; c += 2)
        mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
      tmem_wait_ld32(s + 64);
      tmem_wait_ld32(s + 96);
      // S_t is in registers: the MMA warp may compute the next S_t now
      tc_fence_before();
      mbar_arrive(s_free + t);
      if (masked) {
#pragma unroll
        for (int c = 64; c < 128; ++c)
          if (c >= lim) s[c] = 0xff800000u;
      }
#pragma unroll
      for (int c = 64; c < 128; c += 2)
        mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
      const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c2;
      float alpha = 1.f;
      bool resc = false;
      if (m_tile > m + RESCALE_LOG2 || (m_tile > m && ex2(m_tile - m) > MOVE_SHARE * l)) {
        alpha = ex2(m - m_tile);   // 0 on the first tile (m = -inf)
        resc = (j > 0);
        m = m_tile;
      }
      l *= alpha;
      const float neg_m = (m == -INFINITY) ? 0.f : -m;
      if (L::P_SMEM && j > 0) {
        // PV_t of the previous K/V tile must be done: it reads the P_t buffer
        // and accumulates into O_t, which the rescale below rewrites.  (With P
        // in TMEM, S_t^j was issued after that PV, so s_full already implies
        // it.)
        ok = __all_sync(0xffffffffu, mbar_wait(p_free + t, (j - 1) & 1, wd, ERR_FWD_P_FREE));
        if (!ok) break;
        tc_fence_after();
      }
      const bool rescaled = __any_sync(0xffffffffu, resc);
      if (L::P_SMEM && rescaled) {
        // d = 64: O_t *= alpha now, 32 columns at a time (the S registers are
        // live; with P in shared memory the previous P V has already been
        // waited for above)
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld32(o);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 v =
                fmul2(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2);
            o[i] = __float_as_uint(v.x);
            o[i + 1] = __float_as_uint(v.y);
          }
          tmem_st32(tO + 32 * c, o);
        }
        tmem_wait_st();
      }
      // p = 2^(x - m); exp2_poly_pairs_of_8<D>() pairs in every 8 use the FMA-pipe
      // exp2, the rest MUFU.  P (bf16) goes to this row of the 128B-swizzled
      // K-major P tile: columns 0-63 and 64-127 are two 16 KB regions.
      uint8_t* prow = sP + (L::P_SMEM ? t * 32768 + (r >> 3) * 1024 + (r & 7) * 128 : 0);
      // x = s c2 - m and the row sum in packed pairs (half the issue slots)
      const float2 c22 = make_float2(c2, c2), nm2 = make_float2(neg_m, neg_m);
      float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 x = ffma2(make_float2(__uint_as_float(s[32 * cc + 2 * i]),
                                             __uint_as_float(s[32 * cc + 2 * i + 1])),
                                 c22, nm2);
          float2 pp;
          if ((i & 7) >= 8 - exp2_poly_pairs_of_8<D>())
            pp = ex2_poly2(x);
          else
            pp = make_float2(ex2(x.x), ex2(x.y));
          if (i & 1)
            lb = fadd2(lb, pp);
          else
            la = fadd2(la, pp);
          pk[i] = pack_bf16(pp.x, pp.y);
        }
        if constexpr (L::P_SMEM) {
          uint8_t* reg = prow + (cc >> 1) * 16384;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int ch = (cc & 1) * 4 + k;
            *reinterpret_cast<uint4*>(reg + ((ch ^ (r & 7)) * 16)) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
        } else {
          tmem_st16(tS + 16 * cc, pk);   // P_t over the S_t columns already read
        }
      }
      l += (la.x + la.y) + (lb.x + lb.y);
      // d = 128: O_t *= alpha for the rows whose max moved (the warp does it
      // if any of its rows did) after the exponentials, when the S registers
      // are dead, so the whole row is loaded at once and scaled with packed
      // multiplies; the P V product of this tile is released only afterwards.
      if (!L::P_SMEM && rescaled) {
        uint32_t o[D];
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + 32 * c, o + 32 * c);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_wait_ld32(o + 32 * c);
#pragma unroll
        for (int i = 0; i < D; i += 2) {
          const float2 v =
              fmul2(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), a2);
          o[i] = __float_as_uint(v.x);
          o[i + 1] = __float_as_uint(v.y);
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_st32(tO + 32 * c, o + 32 * c);
      }
      if constexpr (L::P_SMEM)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      else
        tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full + t);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(p_free + t, (n - 1) & 1, wd, ERR_FWD_O_DONE));
      if (ok) {
        tc_fence_after();
        const bool row_ok = qrow < len;
        // block-sparse: a row whose allowed tiles hold no key has l = 0 and
        // an all-zero O accumulator; it gets O = 0 and LSE = -inf
        const bool no_keys = SPARSE && !(l > 0.f);
        const float inv_l = no_keys ? 0.f : 1.f / l;
        const long tok = (p.cu_seqlens != nullptr) ? (long)seq_start + qrow
                                                    : (long)b * p.N + qrow;
        __nv_bfloat16* orow = p.o + (tok * p.Hq + h) * (long)D;
        // optional second output: the bf16 rounding residual of O, so that
        // the backward can form D = rowsum(dO o O) from ~16-bit O
        __nv_bfloat16* lorow = (p.o_lo != nullptr) ? p.o_lo + (tok * p.Hq + h) * (long)D : nullptr;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld32(o);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv_l,
                              __uint_as_float(o[2 * i + 1]) * inv_l);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            if (lorow != nullptr) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16_residual(__uint_as_float(o[2 * i]) * inv_l,
                                           __uint_as_float(o[2 * i + 1]) * inv_l, pk[i]);
              uint4* dlo = reinterpret_cast<uint4*>(lorow + 32 * c);
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4)
                dlo[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            }
          }
        }
        if (row_ok) {
          const float lse = no_keys ? -INFINITY : (m + log2f(l)) * 0.69314718055994530942f;
          const long li = (p.cu_seqlens != nullptr) ? (long)h * p.total + seq_start + qrow
                                                    : ((long)b * p.Hq + h) * p.N + qrow;
          p.lse[li] = lse;
        }
      }
    } else if (SPARSE && n == 0 && qrow < len) {
      // no tile allowed for either Q tile of this CTA: nothing was computed
      const long tok = (long)b * p.N + qrow;
      uint4* dst = reinterpret_cast<uint4*>(p.o + (tok * p.Hq + h) * (long)D);
#pragma unroll 1
      for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0u, 0u, 0u, 0u);
      if (p.o_lo != nullptr) {
        uint4* dlo = reinterpret_cast<uint4*>(p.o_lo + (tok * p.Hq + h) * (long)D);
#pragma unroll 1
        for (int v4 = 0; v4 < D / 8; ++v4) dlo[v4] = make_uint4(0u, 0u, 0u, 0u);
      }
      p.lse[((long)b * p.Hq + h) * p.N + qrow] = -INFINITY;
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
