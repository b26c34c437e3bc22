// fa_bwd.cu - backward of exact attention for sm_100a, by recomputation ("xinc.fun archive
// 235", section 7: the backward recomputes the local scores from the saved inputs and a few
// per-row statistics instead of reading an N x N matrix).
//
// With S = scale Q K^T, P = softmax(S) and the saved LSE_i = ln sum_j exp(S_ij):
//   P_ij = exp(S_ij - LSE_i),  dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO o O),
//   dS = P o (dP - D_i),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels:
//   K2 fa_bwd_pre   per query row: D_i and LSE_i * log2(e), stored per 64-row query tile as
//                   [64 x LSE2 | 64 x D] (rows past N get LSE2 = +inf, D = 0, i.e. P = 0), and
//                   zeroes the fp32 dQ accumulator.  Memory-bound.
//   K3 fa_bwd_main  one CTA per (head, 128-key tile j); K_j and V_j stay in shared memory and
//                   the 64-row query tiles i stream through a 3-stage TMA ring.  Per tile:
//                     S^T  = K_j Q_i^T          (tcgen05, TMEM)
//                     dP^T = V_j dO_i^T         (tcgen05, TMEM)
//                     P^T  = exp2(S^T * scale*log2e - LSE2_i)          (registers -> TMEM)
//                     dV  += P^T dO_i           (tcgen05, A = P^T from TMEM)
//                     dS^T = P^T o (dP^T - D_i)                         (registers -> smem)
//                     dK  += dS^T Q_i           (tcgen05, A = dS^T from shared memory)
//                     dQ_i^T = K_j^T dS^T        (tcgen05, B = dS^T from shared memory)
//                   and dQ_i^T is added into the fp32 accumulator by a TMA reduce-add from a
//                   shared staging slice.  TMEM columns: S^T [0,64), P^T x2 [64,128), the
//                   dP^T / dQ^T pair x2 [128,256), dV [256,384), dK [384,512).
//   K4 fa_bwd_post  dQ = scale * accumulator, rounded to bf16.
#include "fa_debug.cuh"
#include "fa_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda_bf16.h>

#include <algorithm>
#include <climits>
#include <cmath>

namespace fa {

using namespace ptx;

namespace {
constexpr float kLog2e = 1.4426950408889634074f;
}

// ------------------------------------------------------------------ K2
// One 64-row query tile per block iteration (grid-stride over the B*H*Tq tiles), four threads
// per row.  Thread q of a row reads the row's 16-byte pieces q, q + 4, q + 8, ... of O and dO,
// so that a row's four threads read 64 contiguous bytes per load instruction and each thread
// has D / 16 loads in flight, and zeroes the fp32 dQ accumulator row the same way.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ ld,
                                                         float* __restrict__ dq_acc, int* __restrict__ work,
                                                         int BH, int N, int Tq) {
  constexpr int PIECES = D / 32;  // 16-byte pieces of a bf16 row per thread
  if (blockIdx.x == 0 && threadIdx.x < 2) work[threadIdx.x] = 0;  // the key-tile kernel's work counter
  const int r = threadIdx.x >> 2;  // row within the tile
  const int q = threadIdx.x & 3;
  const long long tiles = (long long)BH * Tq;
  for (long long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const int bh = (int)(tile / Tq);
    const int qp = (int)(tile % Tq) * 64 + r;
    float dsum = 0.f, l2 = INFINITY;
    if (qp < N) {
      const size_t row = (size_t)bh * N + qp;
      const uint4* po = reinterpret_cast<const uint4*>(o + row * D);
      const uint4* pg = reinterpret_cast<const uint4*>(dO + row * D);
      uint4 ov[PIECES], gv[PIECES];
#pragma unroll
      for (int m = 0; m < PIECES; ++m) {
        ov[m] = po[q + 4 * m];
        gv[m] = pg[q + 4 * m];
      }
      const float L = lse[row];
      if (dq_acc) {
        float4* pz = reinterpret_cast<float4*>(dq_acc + row * D);
#pragma unroll
        for (int m = 0; m < 2 * PIECES; ++m) pz[q + 4 * m] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int m = 0; m < PIECES; ++m) {
        const uint32_t ow[4] = {ov[m].x, ov[m].y, ov[m].z, ov[m].w};
        const uint32_t gw[4] = {gv[m].x, gv[m].y, gv[m].z, gv[m].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[e]));
          const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[e]));
          dsum = fmaf(of.x, gf.x, fmaf(of.y, gf.y, dsum));
        }
      }
      l2 = (L == -INFINITY) ? INFINITY : L * kLog2e;  // a row with no visible key gets P = 0
    }
    dsum += __shfl_xor_sync(0xffffffffu, dsum, 1);
    dsum += __shfl_xor_sync(0xffffffffu, dsum, 2);
    if (q == 0) {
      float* t = ld + tile * 128;
      t[r] = l2;
      t[64 + r] = dsum;
    }
  }
}

// ------------------------------------------------------------------ K4
__global__ void __launch_bounds__(256) fa_bwd_post_kernel(const float4* __restrict__ acc,
                                                          uint2* __restrict__ dq, long long n4,
                                                          float scale) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const float4 a = acc[i];
    uint2 r;
    r.x = pack_bf16(a.x * scale, a.y * scale);
    r.y = pack_bf16(a.z * scale, a.w * scale);
    dq[i] = r;
  }
}

// Accumulator add for the sequence-sharded backward: acc += x, fp32, 16 bytes per thread.
__global__ void __launch_bounds__(256) fa_acc_add_kernel(float4* __restrict__ acc, const float4* __restrict__ x,
                                                         long long n4) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    float4 a = acc[i];
    const float4 b = x[i];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    acc[i] = a;
  }
}

// ------------------------------------------------------------------ K3
template <int D_>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr int NBOX = D / 64;       // 64-column (128-byte) swizzle boxes per row
  static constexpr int BQ = 64;             // query rows per step
  static constexpr int NSQ = 3;             // Q/dO ring stages
  static constexpr int KT = 128 * D * 2;    // bytes of K_j (or V_j)
  static constexpr int QT = BQ * D * 2;     // bytes of Q_i (or dO_i)
  static constexpr int LDB = 512;           // LSE2 + D of one query tile
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = KT;
  static constexpr int ST_OFF = 2 * KT;     // stage s: [Q_i | dO_i], 2*QT bytes
  static constexpr int ST_BYTES = 2 * QT;
  static constexpr int DS_OFF = ST_OFF + NSQ * ST_BYTES;  // dS^T, two buffers of 128 x 64 bf16
  static constexpr int DS_BYTES = 128 * BQ * 2;
  // d = 64: 16 KB of zeros after the dS^T buffers, the rows d = 64..127 of the dQ^T MMA's A
  // operand, so that dQ^T keeps M = 128 (its TMEM lanes 64..127 come out exactly 0)
  static constexpr int Z_OFF = DS_OFF + 2 * DS_BYTES;
  static constexpr int Z_BYTES = D == 64 ? 128 * 64 * 2 : 0;
  static constexpr int DQS_OFF = Z_OFF + Z_BYTES;   // dQ staging: 4 warps x [rows][32 d] fp32
  static constexpr int DQS_WARP = (BQ - kBwdDqRedRows) * 32 * 4;
  static constexpr int LD_OFF = DQS_OFF + 4 * DQS_WARP;
  static constexpr int BAR_OFF = LD_OFF + NSQ * LDB;
  // kv_full, qd_full[3], qd_empty[3], s_full, s_free, dp_full[2], p_ready[2], ds_ready[2],
  // dq_full[2], dq_free[2], ds_free[2], kv_done, dv_done[2], sc_done, item_full[2],
  // item_empty[2], dv_free, dk_free, gr_done
  static constexpr int NBAR = 1 + 2 * NSQ + 25;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;  // MISC: TMEM base, abort flag, item slots[2]
  static constexpr int THREADS = 480;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns (a 512-column allocation always starts at column 0, lane 0)
  // S^T has one buffer [0, 64), released as soon as the compute warps have loaded it.  P^T
  // (bf16, two per column) is double-buffered: tile n's at [T_P + 32 (n & 1), +32).  So is the
  // gradient pair at T_G: tile n's dP^T goes to [T_G + 64 (n & 1), +64), and once dS_n has
  // been computed from it, tile n's dQ^T goes to the same columns.
  static constexpr uint32_t T_S = 0, T_P = 64, T_G = 128, T_DV = 256, T_DK = 384;
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BQ, false, false);   // S^T, dP^T
  static constexpr uint32_t IDESC_KV = idesc_bf16(128, D, false, true);    // dV, dK (B MN-major)
  static constexpr uint32_t IDESC_Q = idesc_bf16(128, BQ, true, true);     // dQ^T
};

// Roles (480 threads), in a persistent CTA (at most one per SM) that runs item after item:
//   warps 0-3   compute warpgroup 0: P^T and dS^T for query columns [0, 32)  (one key row each)
//   warps 4-7   compute warpgroup 1: the same for query columns [32, 64)
//   warps 8-11  dQ^T drain: TMEM -> shared staging -> TMA reduce-add into the fp32 accumulator;
//               after each item, its epilogue: dV and scale * dK out of TMEM to global memory
//   warp 12     score issuer: S^T and dP^T (whole warp, one elected lane issues)
//   warp 13     TMA producer and work fetch (whole warp, one elected lane issues)
//   warp 14     gradient issuer: dV, dK and dQ^T
// Two issuers, so that neither kind of product waits behind the other's barriers and commits.
// Their products share no accumulator; the one overwrite that crosses them (dP^T of tile t+1
// into the columns whose dQ^T of tile t-1 the drain reads) waits for dq_free, and a Q/dO
// stage is released when both have committed their last use.  P^T of query columns
// [32g, 32g+32) sits at TMEM columns [16g, 16g+16) of the tile's P^T buffer.  dS^T goes to
// shared memory only, where it is the A operand of dK += dS^T Q_i and the B operand of
// dQ^T = K_j^T dS^T.
//
// The schedule keeps the slow chains (scores -> P on the compute warps, P -> dV on the tensor
// core) off each other's critical path: with P^T in its own buffers, S_{t+1} is issued as soon
// as the compute warps have loaded S_t into registers, long before they need it, and a P^T
// buffer is rewritten two tiles after its dV.  dP^T and dQ^T share two alternating TMEM
// buffers: dP_t is dead once dS_t is computed, so dQ_t takes its columns, and dP_{t+1} goes to
// the other buffer as soon as the drain has read dQ_{t-1} from it (without dQ: as soon as
// dS_{t-1} is computed), so it is done before the compute warps need it instead of being
// issued after dS_t.  Tiles are counted over all the CTA's items, so every buffer and phase
// carries from one item into the next: an item's first scores are issued while the previous
// item's last gradients are still in the tensor pipe, and its epilogue (on the drain warps)
// runs while the next item's first tiles are computed; only K_j and V_j wait for the previous
// item's last products.
// WITH_DQ = false: dK and dV only (dQ comes from fa_bwd_dq_kernel): no dQ^T MMA, no drain.
// The dQ^T MMA puts d on the M dimension, which is 128 TMEM lanes; at D = 64 its A operand
// (K_j^T) is extended by 64 rows of zeros in shared memory, so rows 64..127 of dQ^T are 0 and
// only the first two drain warps have anything to add.
template <int D, bool WITH_DQ>
__global__ void __launch_bounds__(480, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                       const __grid_constant__ CUtensorMap tmdQ, const BwdArgs a, const int Tk,
                       const int Tq) {
  static_assert(D == 64 || D == 128, "head dimension");
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work list: the (head, key tile) items, heads in groups of a.group, every head's heaviest
  // key tile first within a group (see fa_fwd_kernel for the trade-off).  A CTA starts with item
  // blockIdx.x and then takes the next unclaimed one from the work counter, so that items go to
  // whichever CTA is about to run dry, in list order, without a CTA launch per item.
  const int items = a.BH * Tk;
  struct Item {
    int bh, j, i0, count;
  };
  auto decode = [&](int idx) -> Item {
    Item w;
    const int per_group = a.group * Tk;
    const int g0 = idx / per_group * a.group;
    const int gn = min(a.group, a.BH - g0);
    const int r = idx - idx / per_group * per_group;
    w.bh = g0 + r % gn;
    w.j = r / gn;                       // keys [128 j, +128)
    w.i0 = a.causal ? 2 * w.j : 0;      // first query tile with a visible pair
    w.count = max(0, Tq - w.i0);
    return w;
  };

  const uint32_t bar = sb + C::BAR_OFF;
  const uint32_t kv_full = bar;
  auto qd_full = [&](int s) { return bar + 8u * (1 + s); };
  auto qd_empty = [&](int s) { return bar + 8u * (1 + C::NSQ + s); };
  // barrier block after the ring's: s_full 0 | s_free 8 | dp_full[2] 16, 24 | p_ready[2] 32, 40 |
  // dq_full[2] 48, 56 | dq_free[2] 64, 72 | ds_free[2] 80, 88 | kv_done 96 | dv_done[2] 104, 112 |
  // sc_done 120 | ds_ready[2] 128, 136 | item_full[2] 144, 152 | item_empty[2] 160, 168 |
  // dv_free 176 | dk_free 184 | gr_done 192: twenty-five 8-byte barriers
  static_assert(C::NBAR == 1 + 2 * C::NSQ + 25, "barrier block layout");
  const uint32_t bar2 = bar + 8u * (1 + 2 * C::NSQ);
  const uint32_t s_full = bar2;      // S_t complete
  const uint32_t s_free = bar2 + 8;  // S_t loaded by both compute warpgroups
  // Tiles are counted over all items of the CTA (t); buffer b = t & 1.  The gradient-pair
  // buffers, one barrier each way: dP_t complete (dp_full), dQ_t complete (dq_full), dQ_t read
  // by the drain (dq_free)
  auto dp_full = [&](int b) { return bar2 + 16 + 8u * b; };
  // P_t and dS_t ready, one barrier per P^T / dS^T buffer: a tile's arrival on a buffer needs the
  // previous tile of that buffer consumed by both issuers, so no waiter ever falls two phases
  // behind
  auto p_ready = [&](int b) { return bar2 + 32 + 8u * b; };
  auto ds_ready = [&](int b) { return bar2 + 128 + 8u * b; };
  auto dq_full = [&](int b) { return bar2 + 48 + 8u * b; };
  auto dq_free = [&](int b) { return bar2 + 64 + 8u * b; };
  auto ds_free = [&](int b) { return bar2 + 80 + 8u * b; };
  const uint32_t kv_done = bar2 + 96;                         // an item's last products have completed
  auto dv_done = [&](int b) { return bar2 + 104 + 8u * b; };  // dV_t (t & 1 == b) has completed
  const uint32_t sc_done = bar2 + 120;                        // the score issuer's products, at exit
  auto item_full = [&](int s) { return bar2 + 144 + 8u * s; };   // item slot s published
  auto item_empty = [&](int s) { return bar2 + 160 + 8u * s; };  // item slot s read by every role
  const uint32_t dv_free = bar2 + 176;  // the epilogue has read an item's dV from TMEM
  const uint32_t dk_free = bar2 + 184;  // ... and its dK
  const uint32_t gr_done = bar2 + 192;  // the gradient issuer's products, at exit
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gb + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + C::MISC_OFF + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(gb + C::MISC_OFF + 8);
  const WaitCtx wc{abort_flag, a.status};
  constexpr int kConsumerWarps = 14;  // every warp but the producer reads each item slot

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::NSQ; ++s) {
      mbar_init(qd_full(s), 1);
      mbar_init(qd_empty(s), 2);  // released by both issuers
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(dp_full(b), 1);
      mbar_init(p_ready(b), 256);
      mbar_init(ds_ready(b), 256);
      mbar_init(dq_full(b), 1);
      mbar_init(dq_free(b), D);  // the drain warps that hold dQ^T rows: one per 32 of d
      mbar_init(ds_free(b), 1);
      mbar_init(dv_done(b), 1);
      mbar_init(item_full(b), 1);
      mbar_init(item_empty(b), kConsumerWarps);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    mbar_init(kv_done, 1);
    mbar_init(sc_done, 1);
    mbar_init(gr_done, 1);
    mbar_init(dv_free, 128);
    mbar_init(dk_free, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(sb + C::MISC_OFF, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (C::Z_BYTES > 0) {
    for (int i = threadIdx.x; i < C::Z_BYTES / 16; i += C::THREADS)
      reinterpret_cast<uint4*>(gb + C::Z_OFF)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();  // visible to the tensor core's reads
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // All TMEM addresses below are compile-time column offsets from address 0.
  if (*tmem_slot != 0u) {
    if (threadIdx.x == 0) atomicOr(a.status, FA_DEV_TMEM_BASE);
    *abort_flag = 1;
  }
  const uint32_t tmem = 0u;

  // Item k of this CTA, as published by the producer in slot k & 1 (a consumer warp's lane 0
  // releases the slot once every lane has read it); -1 when the wait gave up.
  auto next_item = [&](int k) -> int {
    if (!__all_sync(0xffffffffu, mbar_wait(item_full(k & 1), (k >> 1) & 1, wc))) return -1;
    const int idx = item_slot[k & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(item_empty(k & 1));
    return idx;
  };

  if (warp == 13) {
    // ------------------------------------------------------------ TMA producer (whole warp)
    // Per item: publish it, load its first Q/dO tile, then K_j and V_j as soon as every product
    // of the previous item that reads them has completed (kv_done), then its other Q/dO tiles,
    // then claim the next item.  The last slot published holds an index past the list, where
    // every role stops.
    bool ok = !*abort_flag;
    int t = 0;      // Q/dO tiles issued, over all items
    int kv_k = -1;  // last item whose K/V load was issued
    if (ok) {
      if (elect_one()) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmdO);
      }
      const uint64_t keep = policy_evict_last();
      const uint64_t once = policy_evict_first();
      int idx = (int)blockIdx.x;
      for (int k = 0;; ++k) {
        if (k >= 2 && !(ok = __all_sync(0xffffffffu, mbar_wait(item_empty(k & 1), ((k >> 1) & 1) ^ 1, wc))))
          break;
        if (lane == 0) {
          item_slot[k & 1] = idx;
          mbar_arrive(item_full(k & 1));
        }
        if (idx >= items) break;
        const Item w = decode(idx);
        FA_DBG(if (!dbg_check(w.bh < a.BH && w.j >= 0 && w.j < Tk && w.i0 >= 0, a.status)) {
          *abort_flag = 1;
          ok = false;
          break;
        })
        auto load_tile = [&](int n) -> bool {
          const int s = t % C::NSQ;
          const int i = w.i0 + n;
          if (!__all_sync(0xffffffffu, mbar_wait(qd_empty(s), ((t / C::NSQ) & 1) ^ 1, wc))) return false;
          FA_DBG(if (!dbg_check(i < Tq && C::BQ * i < a.N &&
                                    ((size_t)w.bh * Tq + i + 1) * 128 <= (size_t)a.BH * Tq * 128, a.status)) {
            *abort_flag = 1;
            return false;
          })
          mbar_arrive_expect_tx_e(qd_full(s), 2 * C::QT + C::LDB);
          const uint32_t st = sb + C::ST_OFF + s * C::ST_BYTES;
          for (int b = 0; b < C::NBOX; ++b) {
            tma_load_3d_e(st + b * 8192, &tmQ, qd_full(s), 64 * b, C::BQ * i, w.bh, keep);
            tma_load_3d_e(st + C::QT + b * 8192, &tmdO, qd_full(s), 64 * b, C::BQ * i, w.bh, keep);
          }
          bulk_load_e(sb + C::LD_OFF + s * C::LDB, a.ld + ((size_t)w.bh * Tq + i) * 128, C::LDB, qd_full(s));
          ++t;
          return true;
        };
        int n = 0;
        if (w.count > 0 && !(ok = load_tile(n++))) break;
        if (k >= 1 && !(ok = __all_sync(0xffffffffu, mbar_wait(kv_done, (k - 1) & 1, wc)))) break;
        mbar_arrive_expect_tx_e(kv_full, 2 * C::KT);
        for (int b = 0; b < C::NBOX; ++b) {
          tma_load_3d_e(sb + C::K_OFF + b * 16384, &tmK, kv_full, 64 * b, 128 * w.j, w.bh, once);
          tma_load_3d_e(sb + C::V_OFF + b * 16384, &tmV, kv_full, 64 * b, 128 * w.j, w.bh, once);
        }
        kv_k = k;
        for (; n < w.count && ok; ++n) ok = load_tile(n);
        if (!ok) break;
        int nxt = 0;
        if (lane == 0) nxt = (int)gridDim.x + atomicAdd(a.work, 1);
        idx = __shfl_sync(0xffffffffu, nxt, 0);
      }
      if (!ok) {  // aborted: let issued copies land before the CTA exits
        if (kv_k >= 0) mbar_wait_drain(kv_full, kv_k & 1);
        for (int back = 1; back <= C::NSQ && t - back >= 0; ++back)
          mbar_wait_drain(qd_full((t - back) % C::NSQ), ((t - back) / C::NSQ) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 12 || warp == 14) {
    // ------------------------------------------------------------ MMA issuers (whole warps)
    // Score issuer:    S_0, dP_0 | [S_t loaded] S_(t+1), [dQ_(t-1) drained] dP_(t+1) | ...
    // Gradient issuer: [P_t ready] dV_t | [dS_t ready] dK_t, dQ_t | ...
    // Every overwrite follows its last reader: S_(t+1) follows the compute warps' load of S_t
    // (s_free), dP_(t+1) follows the drain's read of dQ_(t-1) from the same gradient-pair buffer
    // (dq_free; without dQ, the compute warps' read of dP_(t-1), ds_ready), dQ_t follows the
    // compute warps' read of dP_t (ds_ready), P_(t+2) follows dV_t (dv_done, waited by the
    // compute warps); the dS^T buffer is released after dK_t and dQ_t (ds_free), a Q/dO stage
    // after S_t, dP_t (score issuer) and dV_t, dK_t (gradient issuer).  An item's first dV and
    // dK overwrite the accumulators once the epilogue has read the previous item's (dv_free,
    // dk_free).  The gradient issuer's commit after an item's last tile (kv_done) also covers
    // every score product of the item: each one was consumed by the compute warps before the
    // last dV or dK could start.
    bool ok = !*abort_flag;
    // Base descriptors; each MMA adds its byte offset (see sdesc_add).
    const uint64_t dK_k = sdesc_sw128(sb + C::K_OFF, 16, 1024);        // K_j, K-major (S^T)
    const uint64_t dV_k = sdesc_sw128(sb + C::V_OFF, 16, 1024);        // V_j, K-major (dP^T)
    // K_j, MN-major (dQ^T): rows d = 64..127 one leading-byte offset away (D = 64: the zeros)
    const uint64_t dK_mn = sdesc_sw128(sb + C::K_OFF, D == 128 ? 16384 : C::Z_OFF - C::K_OFF, 1024);
    const uint64_t dQ_k = sdesc_sw128(sb + C::ST_OFF, 16, 1024);       // Q_i, K-major (S^T)
    const uint64_t dO_k = sdesc_sw128(sb + C::ST_OFF + C::QT, 16, 1024);  // dO_i, K-major (dP^T)
    const uint64_t dQ_mn = sdesc_sw128(sb + C::ST_OFF, 8192, 1024);    // Q_i, MN-major (dK)
    const uint64_t dO_mn = sdesc_sw128(sb + C::ST_OFF + C::QT, 8192, 1024);  // dO_i, MN-major (dV)
    const uint64_t dS_k = sdesc_sw128(sb + C::DS_OFF, 16, 1024);       // dS^T, K-major (dK)
    const uint64_t dS_mn = sdesc_sw128(sb + C::DS_OFF, 8192, 1024);    // dS^T, MN-major (dQ^T)
    auto st_off = [&](int t) { return (uint32_t)((t % C::NSQ) * C::ST_BYTES); };
    int t = 0;  // tiles issued, over all items
    if (warp == 12) {
      auto issue_s = [&](int t) {  // S^T = K_j Q_i^T  (K over d)
        const uint32_t so = st_off(t);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32, qo = (k >> 2) * 8192 + (k & 3) * 32;
          mma_ss_e(tmem + C::T_S, sdesc_add(dK_k, ko), sdesc_add(dQ_k, so + qo), C::IDESC_S, k > 0);
        }
        mma_commit_e(s_full);
      };
      auto issue_dp = [&](int t) {  // dP^T = V_j dO_i^T; the last score product of tile t
        const uint32_t so = st_off(t);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32, qo = (k >> 2) * 8192 + (k & 3) * 32;
          mma_ss_e(tmem + C::T_G + 64 * (t & 1), sdesc_add(dV_k, ko), sdesc_add(dO_k, so + qo), C::IDESC_S,
                   k > 0);
        }
        mma_commit_e(dp_full(t & 1));
        mma_commit_e(qd_empty(t % C::NSQ));
      };
      for (int k = 0; ok; ++k) {
        const int idx = next_item(k);
        if (idx < 0) {
          ok = false;
          break;
        }
        if (idx >= items) break;
        const Item w = decode(idx);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(kv_full, k & 1, wc)))) break;
        for (int n = 0; n < w.count; ++n, ++t) {
          if (t >= 1 && !(ok = __all_sync(0xffffffffu, mbar_wait(s_free, (t - 1) & 1, wc)))) break;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(qd_full(t % C::NSQ), (t / C::NSQ) & 1, wc)))) break;
          tc_fence_after();
          issue_s(t);
          if (t >= 2) {  // buffer t & 1 last held tile t-2's dQ^T (or, without dQ, its dP^T)
            const int b2 = t & 1;
            const uint32_t ph = ((t - 2) >> 1) & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(WITH_DQ ? dq_free(b2) : ds_ready(b2), ph, wc)))) break;
            tc_fence_after();
          }
          issue_dp(t);
        }
      }
      mma_commit_e(sc_done);
      if (!ok) mbar_wait_drain(sc_done, 0);
    } else {
      for (int k = 0; ok; ++k) {
        const int idx = next_item(k);
        if (idx < 0) {
          ok = false;
          break;
        }
        if (idx >= items) break;
        const Item w = decode(idx);
        for (int n = 0; n < w.count; ++n, ++t) {
          const int s = t % C::NSQ;
          const int b = t & 1;
          const uint32_t so = st_off(t);
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_ready(b), (t >> 1) & 1, wc)))) break;
          // an item's first dV overwrites the accumulator once the previous item's is read
          if (n == 0 && k >= 1 && !(ok = __all_sync(0xffffffffu, mbar_wait(dv_free, (k - 1) & 1, wc)))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // dV += P^T dO_i  (K over the 64 queries; A = P^T from TMEM)
            mma_ts_e(tmem + C::T_DV, tmem + C::T_P + 32 * b + 8 * kk, sdesc_add(dO_mn, so + kk * 2048),
                     C::IDESC_KV, (n > 0 || kk > 0) ? 1u : 0u);
          mma_commit_e(dv_done(b));
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(ds_ready(b), (t >> 1) & 1, wc)))) break;
          if (n == 0 && k >= 1 && !(ok = __all_sync(0xffffffffu, mbar_wait(dk_free, (k - 1) & 1, wc)))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // dK += dS^T Q_i  (K over the 64 queries; A = dS^T in smem)
            mma_ss_e(tmem + C::T_DK, sdesc_add(dS_k, b * C::DS_BYTES + 32 * kk), sdesc_add(dQ_mn, so + kk * 2048),
                     C::IDESC_KV, (n > 0 || kk > 0) ? 1u : 0u);
          if (WITH_DQ) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dQ_i^T = K_j^T dS^T (K over the 128 keys), over dP_t's columns
              mma_ss_e(tmem + C::T_G + 64 * b, sdesc_add(dK_mn, kk * 2048),
                       sdesc_add(dS_mn, b * C::DS_BYTES + kk * 2048), C::IDESC_Q, kk > 0);
            mma_commit_e(dq_full(b));
          }
          mma_commit_e(ds_free(b));
          mma_commit_e(qd_empty(s));
        }
        if (!ok) break;
        mma_commit_e(kv_done);  // the item's products (dV, dK final in TMEM; K_j, V_j free)
      }
      mma_commit_e(gr_done);
      if (!ok) mbar_wait_drain(gr_done, 0);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ P and dS (one key row each)
    const int g = warp >> 2;          // query columns [32 g, 32 g + 32)
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::T_S + 32 * g;
    const uint32_t tP0 = tmem + lane_off + C::T_P + 16 * g;  // + 32 for odd tiles
    const uint32_t tDP = tmem + lane_off + C::T_G + 32 * g;  // + 64 for odd tiles
    const float cs = a.scale_log2;
    bool ok = !*abort_flag;
    int t = 0;  // tiles processed, over all items
    for (int k = 0; ok; ++k) {
      const int idx = next_item(k);
      if (idx < 0) {
        ok = false;
        break;
      }
      if (idx >= items) break;
      const Item w = decode(idx);
      const int key = 128 * w.j + r;
      const bool key_ok = key < a.N;
      for (int n = 0; n < w.count && ok; ++n, ++t) {
        const int s = t % C::NSQ;
        const int i = w.i0 + n;
        const int b = t & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(qd_full(s), (t / C::NSQ) & 1, wc) &&
                                         mbar_wait(s_full, t & 1, wc));
        if (!ok) break;
        tc_fence_after();
        FA_DBG(if (g == 0 && wq == 0 && lane == 0) dbg_visit(a.visits, a.visits_cap, a.status, w.bh, Tq, i, Tk, w.j);)
        uint32_t sr[32];
        tmem_ld32(tS, sr);
        const float* ldp = reinterpret_cast<const float*>(gb + C::LD_OFF + s * C::LDB) + 32 * g;
        tmem_wait_ld();
        reg_fence(sr);
        tc_fence_before();
        mbar_arrive(s_free);  // S_t is in registers: S_(t+1) may overwrite it
        // causal: query 64 i + 32 g + c sees this key iff it is >= key
        const int first_vis = a.causal ? (key - C::BQ * i - 32 * g) : -1;  // first visible column
        float p[32];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 l2 = *reinterpret_cast<const float4*>(ldp + 4 * c4);
          p[4 * c4 + 0] = ex2(fmaf(__uint_as_float(sr[4 * c4 + 0]), cs, -l2.x));
          p[4 * c4 + 1] = ex2(fmaf(__uint_as_float(sr[4 * c4 + 1]), cs, -l2.y));
          p[4 * c4 + 2] = ex2(fmaf(__uint_as_float(sr[4 * c4 + 2]), cs, -l2.z));
          p[4 * c4 + 3] = ex2(fmaf(__uint_as_float(sr[4 * c4 + 3]), cs, -l2.w));
        }
        if (!key_ok) {
#pragma unroll
          for (int c = 0; c < 32; ++c) p[c] = 0.f;
        } else if (first_vis > 0) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c < first_vis) p[c] = 0.f;
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
        // P^T buffer b last held P_(t-2): wait until dV_(t-2) has read it
        ok = __all_sync(0xffffffffu, mbar_wait(dv_done(b), ((t >> 1) & 1) ^ 1, wc));
        if (!ok) break;
        tc_fence_after();
        tmem_st16(tP0 + 32 * b, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_ready(b));

        ok = __all_sync(0xffffffffu, mbar_wait(dp_full(b), (t >> 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        tmem_ld32(tDP + 64 * b, sr);
        tmem_wait_ld();
        reg_fence(sr);
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 dd = *reinterpret_cast<const float4*>(ldp + 64 + 4 * c4);
          p[4 * c4 + 0] *= __uint_as_float(sr[4 * c4 + 0]) - dd.x;
          p[4 * c4 + 1] *= __uint_as_float(sr[4 * c4 + 1]) - dd.y;
          p[4 * c4 + 2] *= __uint_as_float(sr[4 * c4 + 2]) - dd.z;
          p[4 * c4 + 3] *= __uint_as_float(sr[4 * c4 + 3]) - dd.w;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
        // dS^T row r, query columns [32 g, 32 g + 32), into the shared buffer read by the dK and
        // dQ MMAs (128-byte rows, 16-byte chunks swizzled by the row index)
        ok = __all_sync(0xffffffffu, mbar_wait(ds_free(b), ((t >> 1) & 1) ^ 1, wc));
        if (!ok) break;
        uint8_t* dsrow = gb + C::DS_OFF + b * C::DS_BYTES + r * 128;
#pragma unroll
        for (int c16 = 0; c16 < 4; ++c16) {
          const int chunk = 4 * g + c16;
          *reinterpret_cast<uint4*>(dsrow + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();  // the tcgen05.ld of dP^T is complete before dQ_t may overwrite it
        mbar_arrive(ds_ready(b));
      }
    }
  } else {
    // ------------------------------------------------------------ dQ^T drain and epilogue
    // Drain: one d index per thread.  Epilogue (after each item's last products): one key row
    // per thread, dV then dK out of TMEM, while the other roles start on the next item.
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float* stage = reinterpret_cast<float*>(gb + C::DQS_OFF + wq * C::DQS_WARP);
    const uint32_t stage_s = sb + C::DQS_OFF + wq * C::DQS_WARP;
    // d = 64: dV and dK staged side by side in the warp's slice; d = 128: one after the other
    constexpr bool kBothFit = 2 * C::NBOX * 4096 <= C::DQS_WARP;
    bool ok = !*abort_flag;
    int t = 0;  // tiles drained, over all items
    for (int k = 0; ok; ++k) {
      const int idx = next_item(k);
      if (idx < 0) {
        ok = false;
        break;
      }
      if (idx >= items) break;
      const Item w = decode(idx);
      // rows d >= D of dQ^T are zero (D = 64): their warps have nothing to drain
      for (int n = 0; n < (WITH_DQ && wq * 32 < D ? w.count : 0) && ok; ++n) {
        const int i = w.i0 + n;
        const int b = (t + n) & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(dq_full(b), ((t + n) >> 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        uint32_t v[64];
        const uint32_t tq = tmem + lane_off + C::T_G + 64 * b;
        tmem_ld32(tq, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tq + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        reg_fence(v);
        tc_fence_before();
        mbar_arrive(dq_free(b));  // dP_(t+2) may overwrite these columns now
        // Split between two paths that use different resources: the first kBwdDqRedRows query
        // rows are added with fp32 reductions straight from registers (lane = d, so each row is
        // one coalesced 128-byte request), the rest are staged as a [rows][32 d] fp32 slice in
        // shared memory and added by one TMA reduce-add.
        const int q0 = C::BQ * i;
        FA_DBG(if (!dbg_check(q0 < a.N, a.status)) continue;)
        const int nred = min(kBwdDqRedRows, a.N - q0);
        float* dst = a.dq_acc + ((size_t)w.bh * a.N + q0) * C::D + wq * 32 + lane;
#pragma unroll
        for (int c = 0; c < kBwdDqRedRows; ++c)
          if (c < nred) atomicAdd(dst + (size_t)c * C::D, __uint_as_float(v[c]));
        if (q0 + kBwdDqRedRows < a.N) {
          if (lane == 0) bulk_wait_read0();  // the previous bulk copy has finished reading the staging
          __syncwarp();
#pragma unroll
          for (int c = kBwdDqRedRows; c < 64; ++c) stage[(c - kBwdDqRedRows) * 32 + lane] = __uint_as_float(v[c]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_3d(&tmdQ, stage_s, 32 * wq, q0 + kBwdDqRedRows, w.bh);
            bulk_commit();
          }
        }
      }
      t += w.count;
      if (!ok) break;

      // ---------------------------------------------------------- epilogue of item k: dV, dK
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(kv_done, k & 1, wc)))) break;
      tc_fence_after();
      const int r = wq * 32 + lane;
      const int key = 128 * w.j + r;
      if (a.dk_acc != nullptr) {
        // accumulate mode: add this key row's scale * dK (or dV) into the fp32 accumulator row
        // (acc_overwrite: store it there); this CTA is the only one touching these rows in this
        // call
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const bool is_dk = which == 1;
          const float mul = is_dk ? a.scale : 1.f;
          const uint32_t src = tmem + lane_off + (is_dk ? C::T_DK : C::T_DV);
          float* accrow = (is_dk ? a.dk_acc : a.dv_acc) + ((size_t)w.bh * a.N + key) * C::D;
#pragma unroll 1
          for (int c32 = 0; c32 < C::D; c32 += 32) {
            uint32_t o[32];
            tmem_ld32(src + c32, o);
            tmem_wait_ld();
            reg_fence(o);
            if (c32 + 32 == C::D) {  // every TMEM read of this accumulator is done
              tc_fence_before();
              mbar_arrive(is_dk ? dk_free : dv_free);
            }
            if (key < a.N && a.acc_overwrite) {
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                const bool z = w.count == 0;
                *reinterpret_cast<float4*>(accrow + c32 + 4 * cc) =
                    make_float4(z ? 0.f : __uint_as_float(o[4 * cc + 0]) * mul, z ? 0.f : __uint_as_float(o[4 * cc + 1]) * mul,
                                z ? 0.f : __uint_as_float(o[4 * cc + 2]) * mul, z ? 0.f : __uint_as_float(o[4 * cc + 3]) * mul);
              }
            } else if (key < a.N && w.count > 0) {
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                float4* pa = reinterpret_cast<float4*>(accrow + c32 + 4 * cc);
                float4 g4 = *pa;
                g4.x += __uint_as_float(o[4 * cc + 0]) * mul;
                g4.y += __uint_as_float(o[4 * cc + 1]) * mul;
                g4.z += __uint_as_float(o[4 * cc + 2]) * mul;
                g4.w += __uint_as_float(o[4 * cc + 3]) * mul;
                *pa = g4;
              }
            }
          }
        }
      } else {
        // bf16 rows staged in this warp's slice (128-byte swizzled boxes of 32 rows x 64 d), stored
        // by TMA; the slice's previous bulk copy must have finished reading it
        uint8_t* stg = gb + C::DQS_OFF + wq * C::DQS_WARP;
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const bool is_dk = which == 1;
          const float mul = is_dk ? a.scale : 1.f;
          const uint32_t src = tmem + lane_off + (is_dk ? C::T_DK : C::T_DV);
          const uint32_t base = (is_dk && kBothFit) ? C::NBOX * 4096 : 0;
          if (which == 0 || !kBothFit) {
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
          }
#pragma unroll
          for (int bx = 0; bx < C::NBOX; ++bx) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t o[32];
              tmem_ld32(src + 64 * bx + 32 * h, o);
              tmem_wait_ld();
              reg_fence(o);
              if (w.count == 0) {
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = 0u;
              }
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) {
                uint4 q4;
                q4.x = pack_bf16(__uint_as_float(o[8 * cc + 0]) * mul, __uint_as_float(o[8 * cc + 1]) * mul);
                q4.y = pack_bf16(__uint_as_float(o[8 * cc + 2]) * mul, __uint_as_float(o[8 * cc + 3]) * mul);
                q4.z = pack_bf16(__uint_as_float(o[8 * cc + 4]) * mul, __uint_as_float(o[8 * cc + 5]) * mul);
                q4.w = pack_bf16(__uint_as_float(o[8 * cc + 6]) * mul, __uint_as_float(o[8 * cc + 7]) * mul);
                const int chunk = h * 4 + cc;
                *reinterpret_cast<uint4*>(stg + base + bx * 4096 + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = q4;
              }
            }
          }
          tc_fence_before();
          mbar_arrive(is_dk ? dk_free : dv_free);  // every TMEM read of this accumulator is done
          fence_proxy_async_smem();
          __syncwarp();
          const int row0 = 128 * w.j + 32 * wq;
          if (lane == 0 && row0 < a.N) {
            for (int bx = 0; bx < C::NBOX; ++bx)
              tma_store_3d(is_dk ? &tmdK : &tmdV, stage_s + base + bx * 4096, 64 * bx, row0, w.bh);
            bulk_commit();
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, C::TMEM_COLS);
  }
  // Every CTA has stopped claiming items once all have counted themselves out here: the last
  // one zeroes the work counter for the next launch.
  if (threadIdx.x == 0 && atomicAdd(a.work + 1, 1) == (int)gridDim.x - 1) {
    atomicExch(a.work, 0);
    atomicExch(a.work + 1, 0);
  }
}

// ------------------------------------------------------------------ launchers
static int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  const long long cap = 148LL * 16;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

cudaError_t launch_bwd_pre(const void* o, const void* dO, const float* lse, float* ld, float* dq_acc,
                           int* work, int BH, int N, int d, cudaStream_t stream) {
  const int Tq = (N + 63) / 64;
  const long long tiles = (long long)BH * Tq;
  auto* po = reinterpret_cast<const __nv_bfloat16*>(o);
  auto* pg = reinterpret_cast<const __nv_bfloat16*>(dO);
  if (d == 64)
    fa_bwd_pre_kernel<64><<<grid_for(tiles, 1), 256, 0, stream>>>(po, pg, lse, ld, dq_acc, work, BH, N, Tq);
  else
    fa_bwd_pre_kernel<128><<<grid_for(tiles, 1), 256, 0, stream>>>(po, pg, lse, ld, dq_acc, work, BH, N, Tq);
  return cudaGetLastError();
}

template <int D, bool WITH_DQ>
static cudaError_t launch_bwd_main_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                     const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                                     const CUtensorMap& tdq, const BwdArgs& a, cudaStream_t stream) {
  using C = BwdCfg<D>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  static_assert(C::SMEM > 116 * 1024, "one CTA per SM: each allocates all 512 TMEM columns");
  static bool attr_set[64];  // per device: the attribute outlives the call
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(fa_bwd_main_kernel<D, WITH_DQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int Tk = (a.N + 127) / 128;
  const int Tq = (a.N + 63) / 64;
  const long long items = (long long)a.BH * Tk;
  if (items > INT_MAX / 2) return cudaErrorInvalidValue;
  if (items == 0) return cudaSuccess;
  if (a.work == nullptr) return cudaErrorInvalidValue;
  static int sms[64];  // per device
  if (dev >= 0 && dev < 64 && sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const long long nsm = (dev >= 0 && dev < 64 && sms[dev] > 0) ? sms[dev] : 148;
  const long long grid = std::min(items, nsm);  // persistent: one CTA per SM at most
  BwdArgs b = a;
  FA_DBG(b.visits = debug_visits(1); b.visits_cap = kDebugVisitInts;)
  fa_bwd_main_kernel<D, WITH_DQ><<<(unsigned)grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, tdo, tdk, tdv,
                                                                                    tdq, b, Tk, Tq);
  return cudaGetLastError();
}

cudaError_t launch_bwd_main(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const CUtensorMap& tdk, const CUtensorMap& tdv,
                            const CUtensorMap& tdq, const BwdArgs& a, cudaStream_t stream, bool with_dq) {
  if (d == 64)
    return with_dq ? launch_bwd_main_t<64, true>(tq, tk, tv, tdo, tdk, tdv, tdq, a, stream)
                   : launch_bwd_main_t<64, false>(tq, tk, tv, tdo, tdk, tdv, tdq, a, stream);
  if (d != 128) return cudaErrorNotSupported;
  return with_dq ? launch_bwd_main_t<128, true>(tq, tk, tv, tdo, tdk, tdv, tdq, a, stream)
                 : launch_bwd_main_t<128, false>(tq, tk, tv, tdo, tdk, tdv, tdq, a, stream);
}

cudaError_t launch_acc_add(float* acc, const float* x, long long elems, cudaStream_t stream) {
  const long long n4 = elems / 4;
  fa_acc_add_kernel<<<grid_for(n4, 256), 256, 0, stream>>>(reinterpret_cast<float4*>(acc),
                                                          reinterpret_cast<const float4*>(x), n4);
  return cudaGetLastError();
}

cudaError_t launch_bwd_post(const float* dq_acc, void* dq, long long elems, float scale, cudaStream_t stream) {
  const long long n4 = elems / 4;
  fa_bwd_post_kernel<<<grid_for(n4, 256), 256, 0, stream>>>(reinterpret_cast<const float4*>(dq_acc),
                                                            reinterpret_cast<uint2*>(dq), n4, scale);
  return cudaGetLastError();
}

}  // namespace fa
