// fa_bwd_dq.cu - deterministic dQ for the backward of exact attention (sm_100a).
//
// dQ = scale * dS K with dS = P o (dP - D), P = exp(S - LSE), S = scale Q K^T, dP = dO V^T
// (the recomputation backward of "xinc.fun archive 235", section 7).  Here one CTA owns 128
// query rows and walks the key blocks of 64 keys in order, accumulating dQ in TMEM, so dQ is
// written once per row with a fixed summation order: no atomics, bitwise reproducible.  It
// recomputes S and dP (the main backward kernel, run in its dK/dV-only mode, recomputes them
// too); the pair replaces the main kernel's atomic dQ path when determinism is asked for, and
// serves head dimension 64.
//
// Roles (192 threads): warps 0-3 compute P and dS (one query row per thread, its LSE2 and D in
// registers), warp 4 issues MMAs, warp 5 issues TMA loads.
// TMEM columns: S_b [64 b, 64 b + 64) and dP_b [128 + 64 b, + 64) for key blocks j with
// b = j & 1 (dS_j, bf16, overwrites the first 32 columns of S_b), dQ [256, 256 + d).
#include "fa_debug.cuh"
#include "fa_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda_bf16.h>

#include <cmath>

namespace fa {

using namespace ptx;

template <int D>
struct DqCfg {
  static constexpr int NBOX = D / 64;
  static constexpr int QT = 128 * D * 2;      // Q_i or dO_i (128 rows)
  static constexpr int KT = 64 * D * 2;       // K_j or V_j (64 keys)
  static constexpr int NS = 3;                // K/V ring stages, each [K_j | V_j]
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = QT;
  static constexpr int KV_OFF = 2 * QT;
  static constexpr int ST_BYTES = 2 * KT;
  static constexpr int BAR_OFF = KV_OFF + NS * ST_BYTES;
  // q_full, kv_full[NS], kv_empty[NS], s_full[2], ds_ready[2], dq_done
  static constexpr int NBAR = 1 + 2 * NS + 2 + 2 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  // Launched with at least 116 KB so that two CTAs never share an SM: both would ask for all
  // 512 TMEM columns and the second would stall in tcgen05.alloc (d = 64 needs only ~83 KB).
  static constexpr int SMEM_USED = MISC_OFF + 16 + 1024;
  static constexpr int SMEM = SMEM_USED < 116 * 1024 ? 116 * 1024 : SMEM_USED;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256;
  static constexpr uint32_t IDESC_SP = idesc_bf16(128, 64, false, false);  // S, dP (N = 64 keys)
  static constexpr uint32_t IDESC_DQ = idesc_bf16(128, D, false, true);    // dQ (N = d)
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmdQ, const BwdArgs a, const int Tq128,
                     const int Tq64) {
  using C = DqCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work item: (head, 128 query rows); heavier causal tiles first
  const int bh = blockIdx.x / Tq128;
  const int it = Tq128 - 1 - (blockIdx.x % Tq128);
  const int q0 = 128 * it;
  const int Tk64 = (a.N + 63) >> 6;
  const int nblk = a.causal ? min(Tk64, 2 * it + 2) : Tk64;  // 64-key blocks with a visible key

  const uint32_t bar = sb + C::BAR_OFF;
  const uint32_t q_full = bar;
  auto kv_full = [&](int s) { return bar + 8u * (1 + s); };
  auto kv_empty = [&](int s) { return bar + 8u * (1 + C::NS + s); };
  auto s_full = [&](int b) { return bar + 8u * (1 + 2 * C::NS + b); };
  auto ds_ready = [&](int b) { return bar + 8u * (3 + 2 * C::NS + b); };
  const uint32_t dq_done = bar + 8u * (5 + 2 * C::NS);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gb + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + C::MISC_OFF + 4);
  const WaitCtx wc{abort_flag, a.status};

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(ds_ready(b), 128);
    }
    mbar_init(dq_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(sb + C::MISC_OFF, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*tmem_slot != 0u) {  // TMEM addresses below are column offsets from 0
    if (threadIdx.x == 0) atomicOr(a.status, FA_DEV_TMEM_BASE);
    *abort_flag = 1;
  }
  const uint32_t tmem = 0u;
  FA_DBG(if (!(bh < a.BH && it >= 0 && it < Tq128)) {
    if (threadIdx.x == 0) atomicOr(a.status, FA_DEV_BOUNDS);
    *abort_flag = 1;
  })

  if (warp == 5) {
    // ------------------------------------------------------------ TMA producer (whole warp)
    if (!*abort_flag && nblk > 0) {
      const uint64_t keep = policy_evict_last();
      const uint64_t once = policy_evict_first();
      mbar_arrive_expect_tx_e(q_full, 2 * C::QT);
      for (int b = 0; b < C::NBOX; ++b) {
        tma_load_3d_e(sb + C::Q_OFF + b * 16384, &tmQ, q_full, 64 * b, q0, bh, once);
        tma_load_3d_e(sb + C::DO_OFF + b * 16384, &tmdO, q_full, 64 * b, q0, bh, once);
      }
      int j = 0;
      for (; j < nblk; ++j) {
        const int s = j % C::NS;
        if (!__all_sync(0xffffffffu, mbar_wait(kv_empty(s), ((j / C::NS) & 1) ^ 1, wc))) break;
        FA_DBG(if (!dbg_check(64 * j < a.N, a.status)) {
          *abort_flag = 1;
          break;
        })
        mbar_arrive_expect_tx_e(kv_full(s), C::ST_BYTES);
        const uint32_t st = sb + C::KV_OFF + s * C::ST_BYTES;
        for (int b = 0; b < C::NBOX; ++b) {
          tma_load_3d_e(st + b * 8192, &tmK, kv_full(s), 64 * b, 64 * j, bh, keep);
          tma_load_3d_e(st + C::KT + b * 8192, &tmV, kv_full(s), 64 * b, 64 * j, bh, keep);
        }
      }
      if (j < nblk) {  // aborted: let issued copies land before the CTA exits
        mbar_wait_drain(q_full, 0);
        for (int back = 1; back <= C::NS && j - back >= 0; ++back)
          mbar_wait_drain(kv_full((j - back) % C::NS), ((j - back) / C::NS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer (whole warp)
    // S_{j+1} and dP_{j+1} are issued before waiting for dS_j, so the tensor core works on the
    // next key block while the compute warps turn block j into dS_j.
    if (!*abort_flag && nblk > 0) {
      const uint64_t dQ_k = sdesc_sw128(sb + C::Q_OFF, 16, 1024);
      const uint64_t dO_k = sdesc_sw128(sb + C::DO_OFF, 16, 1024);
      const uint64_t dK_k = sdesc_sw128(sb + C::KV_OFF, 16, 1024);
      const uint64_t dV_k = sdesc_sw128(sb + C::KV_OFF + C::KT, 16, 1024);
      const uint64_t dK_mn = sdesc_sw128(sb + C::KV_OFF, 8192, 1024);
      auto issue_sp = [&](int j) {  // S_j = Q K_j^T, dP_j = dO V_j^T  (K over d)
        const uint32_t so = (uint32_t)((j % C::NS) * C::ST_BYTES);
        const uint32_t b = (uint32_t)(j & 1);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t qo = (k >> 2) * 16384 + (k & 3) * 32, ko = (k >> 2) * 8192 + (k & 3) * 32;
          mma_ss_e(tmem + C::T_S + 64 * b, sdesc_add(dQ_k, qo), sdesc_add(dK_k, so + ko), C::IDESC_SP, k > 0);
        }
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t qo = (k >> 2) * 16384 + (k & 3) * 32, ko = (k >> 2) * 8192 + (k & 3) * 32;
          mma_ss_e(tmem + C::T_DP + 64 * b, sdesc_add(dO_k, qo), sdesc_add(dV_k, so + ko), C::IDESC_SP, k > 0);
        }
        mma_commit_e(s_full(b));
      };
      bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, wc));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(kv_full(0), 0, wc));
      if (ok) {
        tc_fence_after();
        issue_sp(0);
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const int b = j & 1;
        if (j + 1 < nblk) {
          // S/dP buffer b^1 was last read by the compute warps before they released dS_{j-1}
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(kv_full((j + 1) % C::NS), ((j + 1) / C::NS) & 1, wc))))
            break;
          tc_fence_after();
          issue_sp(j + 1);
        }
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(ds_ready(b), (j >> 1) & 1, wc)))) break;
        tc_fence_after();
        const uint32_t so = (uint32_t)((j % C::NS) * C::ST_BYTES);
#pragma unroll
        for (int k = 0; k < 4; ++k)  // dQ += dS_j K_j  (K over the 64 keys)
          mma_ts_e(tmem + C::T_DQ, tmem + C::T_S + 64 * b + 8 * k, sdesc_add(dK_mn, so + k * 2048), C::IDESC_DQ,
                   (j > 0 || k > 0) ? 1u : 0u);
        mma_commit_e(kv_empty(j % C::NS));
      }
      mma_commit_e(dq_done);
      if (!ok) mbar_wait_drain(dq_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P and dS (one query row each)
    const int r = warp * 32 + lane;
    const int qrow = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float cs = a.scale_log2;
    float l2 = INFINITY, dd = 0.f;  // rows past N: P = 0
    if (qrow < Tq64 * 64) {
      const float* t = a.ld + ((size_t)bh * Tq64 + (qrow >> 6)) * 128;
      l2 = t[qrow & 63];
      dd = t[64 + (qrow & 63)];
    }
    bool ok = !*abort_flag;
    for (int j = 0; j < nblk && ok; ++j) {
      const int b = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full(b), (j >> 1) & 1, wc));
      if (!ok) break;
      FA_DBG(if (warp == 0 && lane == 0) dbg_visit(a.visits, a.visits_cap, a.status, bh, Tq128, it, Tk64, j);)
      tc_fence_after();
      uint32_t x[64], y[64];
      tmem_ld32(tmem + lane_off + C::T_S + 64 * b, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
      tmem_ld32(tmem + lane_off + C::T_S + 64 * b + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
      tmem_ld32(tmem + lane_off + C::T_DP + 64 * b, *reinterpret_cast<uint32_t(*)[32]>(&y[0]));
      tmem_ld32(tmem + lane_off + C::T_DP + 64 * b + 32, *reinterpret_cast<uint32_t(*)[32]>(&y[32]));
      tmem_wait_ld();
      reg_fence(x);
      reg_fence(y);
      // keys 64 j + c: visible iff below N and (causal) not after this query
      int lim = a.N - 1 - 64 * j;
      if (a.causal) lim = min(lim, qrow - 64 * j);
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        float p0 = ex2(fmaf(__uint_as_float(x[c]), cs, -l2));
        float p1 = ex2(fmaf(__uint_as_float(x[c + 1]), cs, -l2));
        p0 = (c > lim) ? 0.f : p0 * (__uint_as_float(y[c]) - dd);
        p1 = (c + 1 > lim) ? 0.f : p1 * (__uint_as_float(y[c + 1]) - dd);
        pk[c >> 1] = pack_bf16(p0, p1);
      }
      tmem_st32(tmem + lane_off + C::T_S + 64 * b, pk);  // dS_j (bf16) over the first 32 columns
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_ready(b));
    }
    // ---------------------------------------------------------------- epilogue: dQ
    if (ok && nblk > 0) ok = __all_sync(0xffffffffu, mbar_wait(dq_done, 0, wc));
    if (ok) {
      tc_fence_after();
      uint8_t* stage = gb + C::Q_OFF;  // Q_i is dead once dq_done has fired
#pragma unroll
      for (int bx = 0; bx < C::NBOX; ++bx) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t o[32];
          if (nblk > 0) {
            tmem_ld32(tmem + lane_off + C::T_DQ + 64 * bx + 32 * h, o);
            tmem_wait_ld();
            reg_fence(o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[8 * cc + 0]) * a.scale, __uint_as_float(o[8 * cc + 1]) * a.scale);
            w.y = pack_bf16(__uint_as_float(o[8 * cc + 2]) * a.scale, __uint_as_float(o[8 * cc + 3]) * a.scale);
            w.z = pack_bf16(__uint_as_float(o[8 * cc + 4]) * a.scale, __uint_as_float(o[8 * cc + 5]) * a.scale);
            w.w = pack_bf16(__uint_as_float(o[8 * cc + 6]) * a.scale, __uint_as_float(o[8 * cc + 7]) * a.scale);
            const int chunk = h * 4 + cc;
            *reinterpret_cast<uint4*>(stage + bx * 16384 + r * 128 + ((chunk ^ (r & 7)) << 4)) = w;
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int row0 = q0 + 32 * warp;
      if (lane == 0 && row0 < a.N) {
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_store_3d(&tmdQ, sb + C::Q_OFF + bx * 16384 + warp * 4096, 64 * bx, row0, bh);
        bulk_commit();
        bulk_wait_read0();
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, C::TMEM_COLS);
  }
}

template <int D>
static cudaError_t launch_dq_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a,
                               cudaStream_t stream) {
  using C = DqCfg<D>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  static bool attr_set[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(fa_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int Tq128 = (a.N + 127) / 128;
  const int Tq64 = (a.N + 63) / 64;
  const long long grid = (long long)a.BH * Tq128;
  BwdArgs b = a;
  FA_DBG(b.visits = debug_visits(2); b.visits_cap = kDebugVisitInts;)
  fa_bwd_dq_kernel<D><<<(unsigned)grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, tdo, tdq, b, Tq128, Tq64);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a, cudaStream_t stream) {
  if (d == 64) return launch_dq_t<64>(tq, tk, tv, tdo, tdq, a, stream);
  return launch_dq_t<128>(tq, tk, tv, tdo, tdq, a, stream);
}

}  // namespace fa
