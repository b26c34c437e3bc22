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
//                     S^T  = K_j Q_i^T          (tcgen05, TMEM, two buffers)
//                     dP^T = V_j dO_i^T         (tcgen05, TMEM)
//                     P^T  = exp2(S^T * scale*log2e - LSE2_i)          (registers)
//                     dV  += P^T dO_i           (tcgen05, A = P^T from TMEM)
//                     dS^T = P^T o (dP^T - D_i)                         (registers -> smem)
//                     dK  += dS^T Q_i           (tcgen05, A = dS^T from shared memory)
//                     dQ_i^T = K_j^T dS^T        (tcgen05, B = dS^T from shared memory)
//                   and dQ_i^T is added into the fp32 accumulator (reductions from registers
//                   for half of its rows, TMA reduce-add for the other half).
//                   TMEM columns: S^T x2 [0,128), dP^T [128,192), dQ^T [192,256),
//                   dV [256,384), dK [384,512).
//   K4 fa_bwd_post  dQ = scale * accumulator, rounded to bf16.
#include "fa_debug.cuh"
#include "fa_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda_bf16.h>

#include <cmath>

namespace fa {

using namespace ptx;

namespace {
constexpr float kLog2e = 1.4426950408889634074f;
}

// ------------------------------------------------------------------ K2
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                         const __nv_bfloat16* __restrict__ dO,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ ld,
                                                         float* __restrict__ dq_acc, int BH, int N,
                                                         int Tq) {
  constexpr int V = D / 32;  // columns per lane
  const int lane = threadIdx.x & 31;
  const long long total = (long long)BH * Tq * 64;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < total; row += nw) {
    const int bh = (int)(row / ((long long)Tq * 64));
    const int qp = (int)(row % ((long long)Tq * 64));
    float dsum = 0.f, l2 = INFINITY;
    if (qp < N) {
      const size_t base = ((size_t)bh * N + qp) * D + lane * V;
      if (V == 4) {
        const uint2 ov = *reinterpret_cast<const uint2*>(o + base);
        const uint2 gv = *reinterpret_cast<const uint2*>(dO + base);
        const float2 o01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.x));
        const float2 o23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ov.y));
        const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.x));
        const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv.y));
        dsum = o01.x * g01.x + o01.y * g01.y + o23.x * g23.x + o23.y * g23.y;
      } else {
        const float2 o01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + base));
        const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dO + base));
        dsum = o01.x * g01.x + o01.y * g01.y;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
      const float L = lse[(size_t)bh * N + qp];
      l2 = (L == -INFINITY) ? INFINITY : L * kLog2e;  // a row with no visible key gets P = 0
      if (dq_acc) {
        if (V == 4)
          *reinterpret_cast<float4*>(dq_acc + base) = make_float4(0.f, 0.f, 0.f, 0.f);
        else
          *reinterpret_cast<float2*>(dq_acc + base) = make_float2(0.f, 0.f);
      }
    }
    if (lane == 0) {
      float* t = ld + ((size_t)bh * Tq + (qp >> 6)) * 128;
      t[qp & 63] = l2;
      t[64 + (qp & 63)] = dsum;
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
  // dq_full[2], dq_free[2], ds_free[2], kv_done, dv_done[2], sc_done
  static constexpr int NBAR = 1 + 2 * NSQ + 18;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;
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

// Roles (480 threads):
//   warps 0-3   compute warpgroup 0: P^T and dS^T for query columns [0, 32)  (one key row each)
//   warps 4-7   compute warpgroup 1: the same for query columns [32, 64)
//   warps 8-11  dQ^T drain: TMEM -> shared staging -> TMA reduce-add into the fp32 accumulator
//   warp 12     score issuer: S^T and dP^T (whole warp, one elected lane issues)
//   warp 13     TMA producer (whole warp, one elected lane issues)
//   warp 14     gradient issuer: dV, dK and dQ^T
// Two issuers, so that neither kind of product waits behind the other's barriers and commits.
// Their products share no accumulator; the one overwrite that crosses them (dP^T of tile n+1
// into the columns whose dQ^T of tile n-1 the drain reads) waits for dq_free, and a Q/dO
// stage is released when both have committed their last use.  P^T of query columns
// [32g, 32g+32) sits at TMEM columns [16g, 16g+16) of the tile's P^T buffer.  dS^T goes to
// shared memory only, where it is the A operand of dK += dS^T Q_i and the B operand of
// dQ^T = K_j^T dS^T.
//
// The schedule keeps the slow chains (scores -> P on the compute warps, P -> dV on the tensor
// core) off each other's critical path: with P^T in its own buffers, S_{n+1} is issued as soon
// as the compute warps have loaded S_n into registers, long before they need it, and a P^T
// buffer is rewritten two tiles after its dV.  dP^T and dQ^T share two alternating TMEM
// buffers: dP_n is dead once dS_n is
// computed, so dQ_n takes its columns, and dP_{n+1} goes to the other buffer as soon as the
// drain has read dQ_{n-1} from it (without dQ: as soon as dS_{n-1} is computed), so it is
// done before the compute warps need it instead of being issued after dS_n.
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

  // heads in groups of a.group, every head's heaviest key tile first within a group (see
  // fa_fwd_kernel for the trade-off)
  const int item = (int)blockIdx.x;
  const int per_group = a.group * Tk;
  const int g0 = item / per_group * a.group;
  const int gn = min(a.group, a.BH - g0);
  const int r = item - item / per_group * per_group;
  const int bh = g0 + r % gn;
  const int j = r / gn;  // keys [128 j, +128)
  const int i0 = a.causal ? 2 * j : 0;         // first query tile with a visible pair
  const int count = max(0, Tq - i0);

  const uint32_t bar = sb + C::BAR_OFF;
  const uint32_t kv_full = bar;
  auto qd_full = [&](int s) { return bar + 8u * (1 + s); };
  auto qd_empty = [&](int s) { return bar + 8u * (1 + C::NSQ + s); };
  // barrier block after the ring's: s_full 0 | s_free 8 | dp_full[2] 16, 24 | p_ready[2] 32, 40 |
  // dq_full[2] 48, 56 | dq_free[2] 64, 72 | ds_free[2] 80, 88 | kv_done 96 | dv_done[2] 104, 112 |
  // sc_done 120 | ds_ready[2] 128, 136: eighteen 8-byte barriers
  static_assert(C::NBAR == 1 + 2 * C::NSQ + 18, "barrier block layout");
  const uint32_t bar2 = bar + 8u * (1 + 2 * C::NSQ);
  const uint32_t s_full = bar2;      // S_n complete
  const uint32_t s_free = bar2 + 8;  // S_n loaded by both compute warpgroups
  // The gradient-pair buffers (b = n & 1), one barrier each way: dP_n complete (dp_full),
  // dQ_n complete (dq_full), dQ_n read by the drain (dq_free)
  auto dp_full = [&](int b) { return bar2 + 16 + 8u * b; };
  // P_n and dS_n ready, one barrier per P^T / dS^T buffer (b = n & 1): a tile's arrival on a
  // buffer needs the previous tile of that buffer consumed by both issuers, so no waiter ever
  // falls two phases behind
  auto p_ready = [&](int b) { return bar2 + 32 + 8u * b; };
  auto ds_ready = [&](int b) { return bar2 + 128 + 8u * b; };
  auto dq_full = [&](int b) { return bar2 + 48 + 8u * b; };
  auto dq_free = [&](int b) { return bar2 + 64 + 8u * b; };
  auto ds_free = [&](int b) { return bar2 + 80 + 8u * b; };
  const uint32_t kv_done = bar2 + 96;
  auto dv_done = [&](int b) { return bar2 + 104 + 8u * b; };  // dV_n (n & 1 == b) has completed
  const uint32_t sc_done = bar2 + 120;                        // every score product has completed
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gb + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + C::MISC_OFF + 4);
  const WaitCtx wc{abort_flag, a.status};

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
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    for (int b = 0; b < 2; ++b) {
      mbar_init(ds_free(b), 1);
      mbar_init(dv_done(b), 1);
    }
    mbar_init(kv_done, 1);
    mbar_init(sc_done, 1);
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
  FA_DBG(if (!(bh < a.BH && j >= 0 && j < Tk && i0 >= 0)) {
    if (threadIdx.x == 0) atomicOr(a.status, FA_DEV_BOUNDS);
    *abort_flag = 1;
  })

  if (warp == 13) {
    // ------------------------------------------------------------ TMA producer (whole warp)
    if (!*abort_flag) {
      if (elect_one()) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmdO);
      }
      const uint64_t keep = policy_evict_last();
      const uint64_t once = policy_evict_first();
      mbar_arrive_expect_tx_e(kv_full, 2 * C::KT);
      for (int b = 0; b < C::NBOX; ++b) {
        tma_load_3d_e(sb + C::K_OFF + b * 16384, &tmK, kv_full, 64 * b, 128 * j, bh, once);
        tma_load_3d_e(sb + C::V_OFF + b * 16384, &tmV, kv_full, 64 * b, 128 * j, bh, once);
      }
      int n = 0;
      for (; n < count; ++n) {
        const int s = n % C::NSQ;
        const int i = i0 + n;
        if (!__all_sync(0xffffffffu, mbar_wait(qd_empty(s), ((n / C::NSQ) & 1) ^ 1, wc))) break;
        FA_DBG(if (!dbg_check(i < Tq && C::BQ * i < a.N &&
                                  ((size_t)bh * Tq + i + 1) * 128 <= (size_t)a.BH * Tq * 128, a.status)) {
          *abort_flag = 1;
          break;
        })
        mbar_arrive_expect_tx_e(qd_full(s), 2 * C::QT + C::LDB);
        const uint32_t st = sb + C::ST_OFF + s * C::ST_BYTES;
        for (int b = 0; b < C::NBOX; ++b) {
          tma_load_3d_e(st + b * 8192, &tmQ, qd_full(s), 64 * b, C::BQ * i, bh, keep);
          tma_load_3d_e(st + C::QT + b * 8192, &tmdO, qd_full(s), 64 * b, C::BQ * i, bh, keep);
        }
        bulk_load_e(sb + C::LD_OFF + s * C::LDB, a.ld + ((size_t)bh * Tq + i) * 128, C::LDB, qd_full(s));
      }
      if (n < count) {  // aborted: let issued copies land before the CTA exits
        mbar_wait_drain(kv_full, 0);
        for (int back = 1; back <= C::NSQ && n - back >= 0; ++back)
          mbar_wait_drain(qd_full((n - back) % C::NSQ), ((n - back) / C::NSQ) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 12 || warp == 14) {
    // ------------------------------------------------------------ MMA issuers (whole warps)
    // Score issuer:    S_0, dP_0 | [S_n loaded] S_(n+1), [dQ_(n-1) drained] dP_(n+1) | ...
    // Gradient issuer: [P_n ready] dV_n | [dS_n ready] dK_n, dQ_n | ...
    // Every overwrite follows its last reader: S_(n+1) follows the compute warps' load of S_n
    // (s_free), dP_(n+1) follows the drain's read of dQ_(n-1) from the same gradient-pair buffer
    // (dq_free; without dQ, the compute warps' read of dP_(n-1), ds_ready), dQ_n follows the
    // compute warps' read of dP_n (ds_ready), P_(n+2) follows dV_n (dv_done, waited by the
    // compute warps); the dS^T buffer is released after dK_n and dQ_n (ds_free), a Q/dO stage
    // after S_n, dP_n (score issuer) and dV_n, dK_n (gradient issuer).  The gradient issuer's last commit (kv_done) also covers every score
    // product: each one was consumed by the compute warps before the last dV or dK could start.
    if (!*abort_flag) {
      bool ok = __all_sync(0xffffffffu, mbar_wait(kv_full, 0, wc));
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
      auto st_off = [&](int n) { return (uint32_t)((n % C::NSQ) * C::ST_BYTES); };
      if (warp == 12) {
        auto issue_s = [&](int n) {  // S^T = K_j Q_i^T  (K over d)
          const uint32_t so = st_off(n);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32, qo = (k >> 2) * 8192 + (k & 3) * 32;
            mma_ss_e(tmem + C::T_S, sdesc_add(dK_k, ko), sdesc_add(dQ_k, so + qo), C::IDESC_S, k > 0);
          }
          mma_commit_e(s_full);
        };
        auto issue_dp = [&](int n) {  // dP^T = V_j dO_i^T; the last score product of tile n
          const uint32_t so = st_off(n);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32, qo = (k >> 2) * 8192 + (k & 3) * 32;
            mma_ss_e(tmem + C::T_G + 64 * (n & 1), sdesc_add(dV_k, ko), sdesc_add(dO_k, so + qo), C::IDESC_S,
                     k > 0);
          }
          mma_commit_e(dp_full(n & 1));
          mma_commit_e(qd_empty(n % C::NSQ));
        };
        auto wait_q = [&](int n) {
          return __all_sync(0xffffffffu, mbar_wait(qd_full(n % C::NSQ), (n / C::NSQ) & 1, wc));
        };
        if (ok && count > 0) {
          if ((ok = wait_q(0))) {
            tc_fence_after();
            issue_s(0);
            issue_dp(0);
          }
        }
        for (int n = 0; n + 1 < count && ok; ++n) {
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(s_free, n & 1, wc)))) break;
          if (!(ok = wait_q(n + 1))) break;
          tc_fence_after();
          issue_s(n + 1);
          if (n >= 1) {  // buffer (n+1) & 1 last held tile n-1's dQ^T (or, without dQ, its dP^T)
            const int b1 = (n - 1) & 1;
            const uint32_t ph = ((n - 1) >> 1) & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(WITH_DQ ? dq_free(b1) : ds_ready(b1), ph, wc)))) break;
            tc_fence_after();
          }
          issue_dp(n + 1);
        }
        mma_commit_e(sc_done);
        if (!ok) mbar_wait_drain(sc_done, 0);
      } else {
        for (int n = 0; n < count && ok; ++n) {
          const int s = n % C::NSQ;
          const int b = n & 1;
          const uint32_t so = st_off(n);
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_ready(b), (n >> 1) & 1, wc)))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)  // dV += P^T dO_i  (K over the 64 queries; A = P^T from TMEM)
            mma_ts_e(tmem + C::T_DV, tmem + C::T_P + 32 * b + 8 * k,
                     sdesc_add(dO_mn, so + k * 2048), C::IDESC_KV, (n > 0 || k > 0) ? 1u : 0u);
          mma_commit_e(dv_done(b));
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(ds_ready(b), (n >> 1) & 1, wc)))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)  // dK += dS^T Q_i  (K over the 64 queries; A = dS^T in smem)
            mma_ss_e(tmem + C::T_DK, sdesc_add(dS_k, b * C::DS_BYTES + 32 * k), sdesc_add(dQ_mn, so + k * 2048),
                     C::IDESC_KV, (n > 0 || k > 0) ? 1u : 0u);
          if (WITH_DQ) {
#pragma unroll
            for (int k = 0; k < 8; ++k)  // dQ_i^T = K_j^T dS^T (K over the 128 keys), over dP_n's columns
              mma_ss_e(tmem + C::T_G + 64 * b, sdesc_add(dK_mn, k * 2048),
                       sdesc_add(dS_mn, b * C::DS_BYTES + k * 2048), C::IDESC_Q, k > 0);
            mma_commit_e(dq_full(b));
          }
          mma_commit_e(ds_free(b));
          mma_commit_e(qd_empty(s));
        }
        mma_commit_e(kv_done);
        if (!ok) mbar_wait_drain(kv_done, 0);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ P and dS (one key row each)
    const int g = warp >> 2;          // query columns [32 g, 32 g + 32)
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int key = 128 * j + r;
    const bool key_ok = key < a.N;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::T_S + 32 * g;
    const uint32_t tP0 = tmem + lane_off + C::T_P + 16 * g;  // + 32 for odd query tiles
    const uint32_t tDP = tmem + lane_off + C::T_G + 32 * g;  // + 64 for odd query tiles
    const float cs = a.scale_log2;
    bool ok = !*abort_flag;
    for (int n = 0; n < count && ok; ++n) {
      const int s = n % C::NSQ;
      const int i = i0 + n;
      const int b = n & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(qd_full(s), (n / C::NSQ) & 1, wc) &&
                                       mbar_wait(s_full, n & 1, wc));
      if (!ok) break;
      tc_fence_after();
      FA_DBG(if (g == 0 && wq == 0 && lane == 0) dbg_visit(a.visits, a.visits_cap, a.status, bh, Tq, i, Tk, j);)
      uint32_t sr[32];
      tmem_ld32(tS, sr);
      const float* ldp = reinterpret_cast<const float*>(gb + C::LD_OFF + s * C::LDB) + 32 * g;
      tmem_wait_ld();
      reg_fence(sr);
      tc_fence_before();
      mbar_arrive(s_free);  // S_n is in registers: S_(n+1) may overwrite it
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
      // P^T buffer b last held P_(n-2): wait until dV_(n-2) has read it
      ok = __all_sync(0xffffffffu, mbar_wait(dv_done(b), ((n >> 1) & 1) ^ 1, wc));
      if (!ok) break;
      tc_fence_after();
      tmem_st16(tP0 + 32 * b, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_ready(b));

      ok = __all_sync(0xffffffffu, mbar_wait(dp_full(b), (n >> 1) & 1, wc));
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
      ok = __all_sync(0xffffffffu, mbar_wait(ds_free(b), ((n >> 1) & 1) ^ 1, wc));
      if (!ok) break;
      uint8_t* dsrow = gb + C::DS_OFF + b * C::DS_BYTES + r * 128;
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        const int chunk = 4 * g + c16;
        *reinterpret_cast<uint4*>(dsrow + ((chunk ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();  // the tcgen05.ld of dP^T is complete before dQ_n may overwrite it
      mbar_arrive(ds_ready(b));
    }
  } else {
    // ------------------------------------------------------------ dQ^T drain (one d index each)
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float* stage = reinterpret_cast<float*>(gb + C::DQS_OFF + wq * C::DQS_WARP);
    const uint32_t stage_s = sb + C::DQS_OFF + wq * C::DQS_WARP;
    bool ok = !*abort_flag;
    // rows d >= D of dQ^T are zero (D = 64): their warps have nothing to drain
    for (int n = 0; n < (WITH_DQ && wq * 32 < D ? count : 0) && ok; ++n) {
      const int i = i0 + n;
      const int b = n & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full(b), (n >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[64];
      const uint32_t tq = tmem + lane_off + C::T_G + 64 * b;
      tmem_ld32(tq, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld32(tq + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_ld();
      reg_fence(v);
      tc_fence_before();
      mbar_arrive(dq_free(b));  // dP_(n+2) may overwrite these columns now
      // Split between two paths that use different resources: the first kBwdDqRedRows query
      // rows are added with fp32 reductions straight from registers (lane = d, so each row is
      // one coalesced 128-byte request), the rest are staged as a [rows][32 d] fp32 slice in
      // shared memory and added by one TMA reduce-add.
      const int q0 = C::BQ * i;
      FA_DBG(if (!dbg_check(q0 < a.N, a.status)) continue;)
      const int nred = min(kBwdDqRedRows, a.N - q0);
      float* dst = a.dq_acc + ((size_t)bh * a.N + q0) * C::D + wq * 32 + lane;
#pragma unroll
      for (int c = 0; c < kBwdDqRedRows; ++c)
        if (c < nred) atomicAdd(dst + (size_t)c * C::D, __uint_as_float(v[c]));
      if (q0 + kBwdDqRedRows < a.N) {
        if (lane == 0) bulk_wait_read0();  // the previous reduce has finished reading the staging
        __syncwarp();
#pragma unroll
        for (int c = kBwdDqRedRows; c < 64; ++c) stage[(c - kBwdDqRedRows) * 32 + lane] = __uint_as_float(v[c]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tmdQ, stage_s, 32 * wq, q0 + kBwdDqRedRows, bh);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  // ---------------------------------------------------------------- epilogue: dK, dV
  if (warp < 8) {
    const bool is_dk = warp < 4;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    bool ok = !*abort_flag;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(kv_done, 0, wc));
    if (ok && a.dk_acc != nullptr) {
      // accumulate mode: add this key row's scale * dK (or dV) into the fp32 accumulator row;
      // this CTA is the only one touching these rows in this call
      tc_fence_after();
      const float mul = is_dk ? a.scale : 1.f;
      const uint32_t src = tmem + lane_off + (is_dk ? C::T_DK : C::T_DV);
      const int key = 128 * j + r;
      float* accrow = (is_dk ? a.dk_acc : a.dv_acc) + ((size_t)bh * a.N + key) * C::D;
#pragma unroll 1
      for (int c32 = 0; c32 < C::D; c32 += 32) {
        uint32_t o[32];
        tmem_ld32(src + c32, o);
        tmem_wait_ld();
        reg_fence(o);
        if (key < a.N && count > 0) {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            float4* pa = reinterpret_cast<float4*>(accrow + c32 + 4 * cc);
            float4 g = *pa;
            g.x += __uint_as_float(o[4 * cc + 0]) * mul;
            g.y += __uint_as_float(o[4 * cc + 1]) * mul;
            g.z += __uint_as_float(o[4 * cc + 2]) * mul;
            g.w += __uint_as_float(o[4 * cc + 3]) * mul;
            *pa = g;
          }
        }
      }
    } else if (ok) {
      tc_fence_after();
      const float mul = is_dk ? a.scale : 1.f;
      const uint32_t src = tmem + lane_off + (is_dk ? C::T_DK : C::T_DV);
      uint8_t* stage = gb + C::ST_OFF + (is_dk ? 0 : C::ST_BYTES);  // the Q/dO ring is idle now
#pragma unroll
      for (int bx = 0; bx < C::NBOX; ++bx) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t o[32];
          tmem_ld32(src + 64 * bx + 32 * h, o);
          tmem_wait_ld();
          reg_fence(o);
          if (count == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[8 * cc + 0]) * mul, __uint_as_float(o[8 * cc + 1]) * mul);
            w.y = pack_bf16(__uint_as_float(o[8 * cc + 2]) * mul, __uint_as_float(o[8 * cc + 3]) * mul);
            w.z = pack_bf16(__uint_as_float(o[8 * cc + 4]) * mul, __uint_as_float(o[8 * cc + 5]) * mul);
            w.w = pack_bf16(__uint_as_float(o[8 * cc + 6]) * mul, __uint_as_float(o[8 * cc + 7]) * mul);
            const int chunk = h * 4 + cc;
            *reinterpret_cast<uint4*>(stage + bx * 16384 + r * 128 + ((chunk ^ (r & 7)) << 4)) = w;
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int row0 = 128 * j + 32 * wq;
      if (lane == 0 && row0 < a.N) {
        const uint32_t sbuf = sb + C::ST_OFF + (is_dk ? 0 : C::ST_BYTES);
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_store_3d(is_dk ? &tmdK : &tmdV, sbuf + bx * 16384 + wq * 4096, 64 * bx, row0, bh);
        bulk_commit();
        bulk_wait_read0();
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ launchers
static int grid_for(long long work, int per_block) {
  long long g = (work + per_block - 1) / per_block;
  const long long cap = 148LL * 16;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

cudaError_t launch_bwd_pre(const void* o, const void* dO, const float* lse, float* ld, float* dq_acc,
                           int BH, int N, int d, cudaStream_t stream) {
  const int Tq = (N + 63) / 64;
  const long long rows = (long long)BH * Tq * 64;
  auto* po = reinterpret_cast<const __nv_bfloat16*>(o);
  auto* pg = reinterpret_cast<const __nv_bfloat16*>(dO);
  if (d == 64)
    fa_bwd_pre_kernel<64><<<grid_for(rows, 8), 256, 0, stream>>>(po, pg, lse, ld, dq_acc, BH, N, Tq);
  else
    fa_bwd_pre_kernel<128><<<grid_for(rows, 8), 256, 0, stream>>>(po, pg, lse, ld, dq_acc, BH, N, Tq);
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
  const long long grid = (long long)a.BH * Tk;
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

cudaError_t launch_bwd_post(const float* dq_acc, void* dq, long long elems, float scale, cudaStream_t stream) {
  const long long n4 = elems / 4;
  fa_bwd_post_kernel<<<grid_for(n4, 256), 256, 0, stream>>>(reinterpret_cast<const float4*>(dq_acc),
                                                            reinterpret_cast<uint2*>(dq), n4, scale);
  return cudaGetLastError();
}

}  // namespace fa
