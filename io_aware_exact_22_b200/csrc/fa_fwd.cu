// fa_fwd.cu - fused exact-attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Method: the online softmax of "xinc.fun archive 235", section 7 (running max m, denominator
// l and unnormalised accumulator z per query row, o = z / l at the end), one key block of 128
// keys per step, so that the scores S = scale * Q K^T (section 6) and probabilities P never
// leave the SM.  The running max is kept as a reference value that only moves when a block's
// max exceeds it by more than 2^8 (in base-2 units); z and l are relative to that reference,
// which cancels in z / l (see the two-block merge identities of "Flash Attention",
// special-jiahao.github.io, section 增量求解 softmax), and every exponent stays <= 2^8.
//
// One CTA owns 256 query rows of one (batch, head) as two 128-row tiles and streams the K/V
// blocks through a shared-memory ring.  Roles (352 threads):
//   warps 0-3  softmax warpgroup for query tile 0   (one thread per query row)
//   warps 4-7  softmax warpgroup for query tile 1
//   warp  8    score issuer (one thread): S_t = Q_t K_j^T on the tensor core
//   warp  9    TMA producer (one thread): Q tiles once, then K_0, and K_{j+1} ahead of V_j
//   warp  10   output issuer (one thread): O_t += P_t V_j on the tensor core
// The two kinds of product touch disjoint TMEM columns (S against O) and shared memory (Q, K
// against P, V), so they need no order between them, and with one issuer each a P V is issued
// as soon as its P is written instead of after the other tile's score products: each tile's
// chain per block (softmax, then P V) does not wait on the other tile.
// TMEM (512 columns x 128 lanes, fp32): S_0 [0,128), S_1 [128,256), O_0 [256,256+d),
// O_1 [256+d, 256+2d).  P_t goes to shared memory (bf16 or E4M3, the K-major 128-byte-swizzled
// layout of an MMA A operand), so S_t is free as soon as its softmax warpgroup has loaded it
// into registers: S_t for block j+1 is computed while the softmax of block j runs, and each
// tile's chain per block is its softmax alone rather than S MMA + softmax + PV MMA.
#include "fa_debug.cuh"
#include "fa_internal.cuh"

#include <algorithm>
#include "sm100_ptx.cuh"

#include <cmath>

namespace fa {

using namespace ptx;

// Column pairs (out of every 8 pairs) whose exponential is evaluated on the FMA pipe.  Per
// element and warp, MUFU ex2 occupies its pipe ~8 cycles and the polynomial the FMA pipe
// ~9.3, on top of ~3.6 FMA-pipe cycles of scaling, row sum and packing; the two pipes balance
// at a polynomial share of about 1/4.
constexpr int kPolyPairsOf8 = 2;

// FP8: Q, K, V are E4M3 (one byte per element) and both tile GEMMs run as kind::f8f6f4; P is
// quantised to E4M3 for the PV GEMM.  Softmax, accumulators and the output are as for bf16.
template <int D, bool FP8 = false>
struct FwdCfg {
  static constexpr int EB = FP8 ? 1 : 2;           // bytes per input element
  static constexpr int BOXW = 128 / EB;            // elements per 128-byte swizzle box row
  static constexpr int NBOX = D / BOXW;            // swizzle boxes per row
  static constexpr int TILE = 128 * D * EB;        // bytes of one 128-row input tile
  // K/V ring stages (one K or one V tile each).  K_{j+1} is loaded ahead of V_j, so with three
  // stages K_{j+2} reuses V_{j-1}'s stage and V_{j+1} reuses K_{j+1}'s.
  static constexpr int NS = (TILE == 32768) ? 3 : 8;
  static constexpr int KSTEP = 32 / EB;            // elements of K per MMA (32 bytes)
  static constexpr int PTILE = 128 * 128 * EB;     // bytes of one P tile (128 rows x 128 keys)
  static constexpr int OTILE = 128 * D * 2;        // bytes of one 128-row bf16 output tile
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * TILE;
  static constexpr int P_OFF = KV_OFF + NS * TILE;  // ring and P tiles together stage partial outputs
  static constexpr int BAR_OFF = P_OFF + 2 * PTILE;
  // O staging, tile t at OST_OFF + t * OST_STRIDE: the dead P tile (the Q tiles may already
  // hold the next item's queries), OST_BOXES 64-column boxes of bf16 output at a time (FP8:
  // one, its P tile being half a tile's output; the output then goes in two passes)
  static constexpr int OST_OFF = P_OFF;
  static constexpr int OST_STRIDE = PTILE;
  static constexpr int OST_BOXES = PTILE / 16384;
  // barriers: q_full, q_empty, kv_full[NS], kv_empty[NS], s_full[2], s_free[2], p_full[2],
  // pv_done[2], o_full[2], o_free[2], s_done, pv_end
  static constexpr int NBAR = 2 + 2 * NS + 12 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;  // + slack to align the base to 1024
  static constexpr int THREADS = 352;
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns (a 512-column allocation always starts at column 0, lane 0)
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O0 = 256, T_O1 = 256 + D;
  static constexpr uint32_t IDESC_QK = FP8 ? idesc_e4m3(128, 128, false, false) : idesc_bf16(128, 128, false, false);
  static constexpr uint32_t IDESC_PV = FP8 ? idesc_e4m3(128, D, false, true) : idesc_bf16(128, D, false, true);
  // P is computed as 2^(s c - m + P_SHIFT) and the reference m moves once a block's max exceeds
  // it by more than MOVE (both base 2).  bf16: P <= 2^8.  FP8: P <= 2^8.75 < 448 (the largest
  // E4M3 value) and values down to 2^-17 of the reference term stay representable.
  static constexpr float P_SHIFT = FP8 ? 8.0f : 0.0f;
  static constexpr float MOVE = FP8 ? 0.75f : 8.0f;
};

// PARTIAL: the CTA covers only its split's range of key blocks and writes the normalised
// partial output O_s (fp32) and its LSE_s, to be combined by fa_fwd_merge_kernel.
//
// Work list.  An item is (head bh, block of 256 query rows, key split).  With a.persistent = 0
// every CTA takes one item, in the grouped heaviest-first order (heads in groups of a.group;
// within a group every head's heaviest query block first: group 1 keeps a head's blocks
// together, so its K/V stays in L2, group BH gives the shortest causal tail), and the
// hardware hands the next CTA to the first SM that frees up.  With a.persistent = 1 (whole key
// range, bf16) a grid of at most one CTA per SM walks the list itself: each head's query
// blocks in the order heaviest, lightest, second heaviest, second lightest, ..., so that under
// the causal mask consecutive pairs cost the same, and CTA c takes pairs c, c + grid, ...;
// the next item's Q load and first score products then overlap the current item's last
// blocks and output, and the CTA's setup is paid once.
template <int D, bool PARTIAL, bool FP8 = false>
__global__ void __launch_bounds__(352, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdArgs a) {
  static_assert(!FP8 || (D == 128 && !PARTIAL), "FP8: d = 128, whole key range");
  using C = FwdCfg<D, FP8>;
  constexpr bool kOutInP = !PARTIAL;  // the output is staged in the tile's own P tile
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sb = (raw + 1023u) & ~1023u;
  uint8_t* gb = smem_raw + (sb - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Tk = (a.N + 127) >> 7;
  const int total = a.BH * a.nqb * a.nsplit;  // items (the host checks that this fits an int)
  // list index of this CTA's k-th item, or -1 past its last
  auto item_at = [&](int k) -> int {
    if (!a.persistent) return k == 0 ? (int)blockIdx.x : -1;
    const long long idx = 2 * ((long long)blockIdx.x + (long long)(k >> 1) * gridDim.x) + (k & 1);
    return idx < total ? (int)idx : -1;
  };
  struct Item {
    int bh, qb, split, q0, kb0, n0, n1, nmax, n0g, n1g;
    bool has1;
  };
  auto decode = [&](int idx) -> Item {
    Item w;
    if (a.persistent) {
      w.split = 0;
      w.bh = idx / a.nqb;
      const int p = idx - w.bh * a.nqb;
      w.qb = (p & 1) ? (p >> 1) : a.nqb - 1 - (p >> 1);
    } else {
      w.split = idx % a.nsplit;
      const int item = idx / a.nsplit;
      const int per_group = a.group * a.nqb;
      const int g0 = item / per_group * a.group;  // first head of the group
      const int gn = min(a.group, a.BH - g0);     // heads in the group (the last may be short)
      const int r = item - item / per_group * per_group;
      w.bh = g0 + r % gn;
      w.qb = a.nqb - 1 - r / gn;
    }
    w.q0 = w.qb * 256;
    w.has1 = (w.q0 + 128) < a.N;
    // visible key blocks of each query tile, over the whole key range
    w.n0g = a.causal ? min(Tk, 2 * w.qb + 1) : Tk;
    w.n1g = w.has1 ? (a.causal ? min(Tk, 2 * w.qb + 2) : Tk) : 0;
    // this split's contiguous share [kb0, kb1) of the key blocks, and each tile's count in it
    const int nmaxg = max(w.n0g, w.n1g);
    w.kb0 = (int)((long long)w.split * nmaxg / a.nsplit);
    const int kb1 = (int)((long long)(w.split + 1) * nmaxg / a.nsplit);
    w.n0 = max(0, min(kb1, w.n0g) - w.kb0);
    w.n1 = max(0, min(kb1, w.n1g) - w.kb0);
    w.nmax = max(w.n0, w.n1);
    FA_DBG(if (!dbg_check(w.bh < a.BH && w.qb >= 0 && w.qb < a.nqb && w.split < a.nsplit && kb1 <= Tk, a.status))
               *reinterpret_cast<volatile int*>(gb + C::MISC_OFF + 4) = 1;)
    return w;
  };

  const uint32_t bar = sb + C::BAR_OFF;
  const uint32_t q_full = bar;                                               // Q tiles landed
  const uint32_t q_empty = bar + 8u;                                         // Q tiles read by every S
  auto kv_full = [&](int s) { return bar + 8u * (2 + s); };
  auto kv_empty = [&](int s) { return bar + 8u * (2 + C::NS + s); };
  auto s_full = [&](int t) { return bar + 8u * (2 + 2 * C::NS + t); };    // S_t computed
  auto s_free = [&](int t) { return bar + 8u * (4 + 2 * C::NS + t); };    // S_t loaded by its softmax
  auto p_full = [&](int t) { return bar + 8u * (6 + 2 * C::NS + t); };    // P_t written
  auto pv_done = [&](int t) { return bar + 8u * (8 + 2 * C::NS + t); };   // P_t V_j added into O_t
  auto o_full = [&](int t) { return bar + 8u * (10 + 2 * C::NS + t); };   // O_t of the item complete
  auto o_free = [&](int t) { return bar + 8u * (12 + 2 * C::NS + t); };   // O_t read by the epilogue
  const uint32_t s_done = bar + 8u * (14 + 2 * C::NS);  // every score product issued has completed
  const uint32_t pv_end = bar + 8u * (15 + 2 * C::NS);  // every P V product issued has completed
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gb + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + C::MISC_OFF + 4);
  const WaitCtx wc{abort_flag, a.status};

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(s_free(t), 128);
      mbar_init(p_full(t), 128);
      mbar_init(pv_done(t), 1);
      mbar_init(o_full(t), 1);
      mbar_init(o_free(t), 128);
    }
    mbar_init(s_done, 1);
    mbar_init(pv_end, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(sb + C::MISC_OFF, C::TMEM_COLS);
    tmem_relinquish();
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
  // ring positions within an item of nmax blocks: K_0 first, then K_{j+1} (when there is
  // one) before V_j; every item takes 2 nmax consecutive positions
  auto pos_k = [](int j) { return j == 0 ? 0 : 2 * j - 1; };
  const bool carry = !FP8 && a.carry_o != nullptr;  // rows continue from a carried partial result
  auto pos_v = [](int j, int nmax) { return j + 1 < nmax ? 2 * j + 2 : 2 * j + 1; };

  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer (whole warp)
    if (!*abort_flag) {
      if (elect_one()) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      const uint64_t keep = policy_evict_last();
      int it = 0;  // ring position over all items
      int ni = 0;  // items whose Q tiles were loaded
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int idx = item_at(k);
        if (idx < 0) break;
        const Item w = decode(idx);
        if (w.nmax == 0) continue;
        // the Q tiles are reused once every score product of the previous item has completed
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(q_empty, (ni & 1) ^ 1, wc)))) break;
        const int nq = w.has1 ? 2 : 1;
        mbar_arrive_expect_tx_e(q_full, nq * C::TILE);
        for (int t = 0; t < nq; ++t)
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d_e(sb + C::Q_OFF + t * C::TILE + b * 16384, &tmQ, q_full, C::BOXW * b, w.q0 + 128 * t,
                          w.bh, keep);
        ++ni;
        auto load = [&](const CUtensorMap* m, int j) {
          const int s = it % C::NS;
          const uint32_t ph = (it / C::NS) & 1;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(kv_empty(s), ph ^ 1, wc)))) return;
          FA_DBG(if (!dbg_check(w.kb0 + j >= 0 && 128 * (w.kb0 + j) < a.N, a.status)) {
            *abort_flag = 1;
            ok = false;
            return;
          })
          mbar_arrive_expect_tx_e(kv_full(s), C::TILE);
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_3d_e(sb + C::KV_OFF + s * C::TILE + b * 16384, m, kv_full(s), C::BOXW * b,
                          128 * (w.kb0 + j), w.bh, keep);
          ++it;
        };
        load(&tmK, 0);
        for (int j = 0; j < w.nmax && ok; ++j) {
          if (j + 1 < w.nmax) load(&tmK, j + 1);
          if (ok) load(&tmV, j);
        }
      }
      if (!ok) {  // let copies already issued land before the CTA exits
        if (ni > 0) mbar_wait_drain(q_full, (ni - 1) & 1);
        for (int back = 1; back <= C::NS && it - back >= 0; ++back) {
          const int i2 = it - back;
          mbar_wait_drain(kv_full(i2 % C::NS), (i2 / C::NS) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 8 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers (whole warps)
    if (!*abort_flag) {
      // Base descriptors; each MMA adds its byte offset (see sdesc_add).
      const uint64_t dQ_k = sdesc_sw128(sb + C::Q_OFF, 16, 1024);       // Q tiles, K-major
      const uint64_t dK_k = sdesc_sw128(sb + C::KV_OFF, 16, 1024);      // K stages, K-major
      const uint64_t dV_mn = sdesc_sw128(sb + C::KV_OFF, 16384, 1024);  // V stages, MN-major
      const uint64_t dP_k = sdesc_sw128(sb + C::P_OFF, 16, 1024);       // P tiles, K-major
      auto stage_addr = [&](int it) { return (uint32_t)((it % C::NS) * C::TILE); };
      auto stage_par = [&](int it) { return (uint32_t)((it / C::NS) & 1); };
      auto wait_stage = [&](int it) {
        return __all_sync(0xffffffffu, mbar_wait(kv_full(it % C::NS), stage_par(it), wc));
      };
      bool ok = true;
      int ibase = 0;  // ring position of the item's first load
      if (warp == 8) {
        // S_t for block j, each as soon as K_j has landed and tile t's softmax has loaded the
        // previous S_t (of this item or the one before)
        auto issue_qk = [&](uint32_t dst, uint32_t qoff, uint32_t koff) {
#pragma unroll
          for (int k = 0; k < D / C::KSTEP; ++k) {  // 32 bytes of d per MMA
            const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
            if constexpr (FP8)
              mma_ss_e8(dst, sdesc_add(dQ_k, qoff + off), sdesc_add(dK_k, koff + off), C::IDESC_QK, k > 0);
            else
              mma_ss_e(dst, sdesc_add(dQ_k, qoff + off), sdesc_add(dK_k, koff + off), C::IDESC_QK, k > 0);
          }
        };
        int ni = 0;               // items issued
        int cs[2] = {0, 0};       // S_t products issued, over all items
        for (int kk = 0; ok; ++kk) {
          const int idx = item_at(kk);
          if (idx < 0) break;
          const Item w = decode(idx);
          if (w.nmax == 0) continue;
          const int nt[2] = {w.n0, w.n1};
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(q_full, ni & 1, wc)))) break;
          for (int j = 0; j < w.nmax && ok; ++j) {
            const int itK = ibase + pos_k(j);
            if (!(ok = wait_stage(itK))) break;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (j >= nt[t]) continue;
              if (cs[t] > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(s_free(t), (cs[t] - 1) & 1, wc)))) break;
              tc_fence_after();
              issue_qk(t ? C::T_S1 : C::T_S0, (uint32_t)(t * C::TILE), stage_addr(itK));
              mma_commit_e(s_full(t));
              ++cs[t];
            }
            if (!ok) break;
            mma_commit_e(kv_empty(itK % C::NS));
          }
          if (!ok) break;
          mma_commit_e(q_empty);  // the Q tiles are free once these products have completed
          ibase += 2 * w.nmax;
          ++ni;
        }
        mma_commit_e(s_done);
        if (!ok) mbar_wait_drain(s_done, 0);  // every issued MMA has completed before TMEM is freed
      } else {
        // O_t += P_t V_j, each as soon as V_j has landed and tile t's softmax has written P_t; the
        // first of an item also after the epilogue has read the previous item's O_t
        auto issue_pv = [&](uint32_t dst, uint32_t poff, uint32_t voff, bool acc) {
#pragma unroll
          for (int k = 0; k < 128 / C::KSTEP; ++k) {  // KSTEP keys (32 bytes of P) per MMA
            const uint32_t po = poff + (k >> 2) * 16384 + (k & 3) * 32;
            const uint32_t vo = voff + k * C::KSTEP * 128;
            if constexpr (FP8)
              mma_ss_e8(dst, sdesc_add(dP_k, po), sdesc_add(dV_mn, vo), C::IDESC_PV, (acc || k > 0) ? 1u : 0u);
            else
              mma_ss_e(dst, sdesc_add(dP_k, po), sdesc_add(dV_mn, vo), C::IDESC_PV, (acc || k > 0) ? 1u : 0u);
          }
        };
        int cp[2] = {0, 0};  // P_t consumed, over all items
        int co[2] = {0, 0};  // items whose O_t was completed
        for (int kk = 0; ok; ++kk) {
          const int idx = item_at(kk);
          if (idx < 0) break;
          const Item w = decode(idx);
          if (w.nmax == 0) continue;
          const int nt[2] = {w.n0, w.n1};
          for (int j = 0; j < w.nmax && ok; ++j) {
            const int itV = ibase + pos_v(j, w.nmax);
            if (!(ok = wait_stage(itV))) break;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (j >= nt[t]) continue;
              if (j == 0 && co[t] > 0 &&
                  !(ok = __all_sync(0xffffffffu, mbar_wait(o_free(t), (co[t] - 1) & 1, wc))))
                break;
              if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_full(t), cp[t] & 1, wc)))) break;
              tc_fence_after();
              // the first product of an item accumulates onto a carried O (written by the softmax)
              issue_pv(t ? C::T_O1 : C::T_O0, (uint32_t)(t * C::PTILE), stage_addr(itV), j > 0 || carry);
              mma_commit_e(pv_done(t));
              ++cp[t];
              // whole key range: O_t of this item is complete once this product is (its output is
              // staged in P_t, which no other product reads).  Split outputs are staged in the K/V
              // ring, idle only once every product of the item is done.
              if (kOutInP && j == nt[t] - 1) {
                mma_commit_e(o_full(t));
                ++co[t];
              }
            }
            if (!ok) break;
            mma_commit_e(kv_empty(itV % C::NS));
          }
          if (!ok) break;
          if (!kOutInP) {
#pragma unroll
            for (int t = 0; t < 2; ++t)
              if (nt[t] > 0) {
                mma_commit_e(o_full(t));
                ++co[t];
              }
          }
          ibase += 2 * w.nmax;
        }
        mma_commit_e(pv_end);
        if (!ok) mbar_wait_drain(pv_end, 0);  // every issued MMA has completed before TMEM is freed
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row within the query tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tSrow = tmem + lane_off + 128u * t;
    const uint32_t tOrow = tmem + lane_off + 256u + (uint32_t)(D * t);
    bool ok = !*abort_flag;
    bool store_pending = false;  // this warp's O store may still be reading the P_t rows
    int ns = 0;  // S_t blocks consumed, over all items (s_full phases)
    int np = 0;  // P_t blocks written, over all items (pv_done phases)
    int no = 0;  // items whose O_t this warpgroup wrote out (o_full phases)
    for (int kk = 0; ok; ++kk) {
    const int idx = item_at(kk);
    if (idx < 0) break;
    const Item wk = decode(idx);
    const int bh = wk.bh, qb = wk.qb, split = wk.split, kb0 = wk.kb0;
    (void)qb;
    (void)split;
    const int ntile = t ? wk.n1 : wk.n0;      // blocks of this split
    const int ntile_g = t ? wk.n1g : wk.n0g;  // blocks of the whole key range
    const int qrow = wk.q0 + 128 * t + r;
    if (wk.nmax == 0 || ntile == 0) {
      // this split holds no key block of this tile: an empty partial (weight 0 in the merge)
      if (PARTIAL && !carry && qrow < a.N) a.lse[((size_t)split * a.BH + bh) * a.N + qrow] = -INFINITY;
      continue;
    }
    float cs = a.scale_log2;
    float vmul = 1.f;  // FP8: V's dequantisation factor, applied to O at the end
    if constexpr (FP8) {
      if (a.descale_q) cs *= a.descale_q[bh];
      if (a.descale_k) cs *= a.descale_k[bh];
      if (a.descale_v) vmul = a.descale_v[bh];
    }
    float m_ref = -INFINITY;  // reference max, base-2 scaled units
    float l = 0.f;
    if (carry) {
      // Continue from a partial result over other keys ([jiahao] 增量求解 softmax: the blocks'
      // sums and outputs rescaled to a common reference): its LSE is the reference, the sum
      // relative to it is 1 and O_t starts as its normalised output, so the block loop below
      // carries on as if those keys had come first.  A row that has seen no key starts empty.
      const float L = qrow < a.N ? a.carry_lse[(size_t)bh * a.N + qrow] : -INFINITY;
      const bool has = L > -INFINITY;
      if (has) {
        m_ref = L * 1.4426950408889634074f;
        l = 1.f;
      }
      const float* src = a.carry_o + ((size_t)bh * a.N + (has ? qrow : 0)) * D;
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t ov[32];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 f = has ? *reinterpret_cast<const float4*>(src + cc + 4 * e4) : make_float4(0.f, 0.f, 0.f, 0.f);
          ov[4 * e4 + 0] = __float_as_uint(f.x);
          ov[4 * e4 + 1] = __float_as_uint(f.y);
          ov[4 * e4 + 2] = __float_as_uint(f.z);
          ov[4 * e4 + 3] = __float_as_uint(f.w);
        }
        tmem_st32(tOrow + cc, ov);
      }
      tmem_wait_st();
    }

    for (int j = 0; j < ntile && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full(t), ns & 1, wc));
      ++ns;
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(tSrow + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tSrow + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tSrow + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(tSrow + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_wait_ld();
      reg_fence(sr);
      tc_fence_before();
      mbar_arrive(s_free(t));  // S_t may now be overwritten by the next block's scores
      float x[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sr[c]);
      const int jg = kb0 + j;                 // key block index in the whole key range
      FA_DBG(if (wq == 0 && lane == 0) dbg_visit(a.visits, a.visits_cap, a.status, bh, (a.N + 127) >> 7,
                                                 2 * qb + t, Tk, jg);)
      const bool edge = (jg == ntile_g - 1);  // the only block that can hold the diagonal or the tail
      // P_t row r in shared memory: 16-byte chunks g of the 128-byte-swizzled K-major layout (64
      // bf16 or 128 E4M3 keys per 128-byte box row), each stored as soon as its four 32-bit
      // words are packed (word indices are compile-time constants in the unrolled loops)
      uint8_t* prow = gb + C::P_OFF + t * C::PTILE + r * 128;
      uint32_t cw[4];
      auto put_word = [&](int w, uint32_t v) {
        cw[w & 3] = v;
        if ((w & 3) == 3) {
          const int g = w >> 2;
          *reinterpret_cast<uint4*>(prow + (g >> 3) * 16384 + (((g & 7) ^ (r & 7)) << 4)) =
              make_uint4(cw[0], cw[1], cw[2], cw[3]);
        }
      };

      // Exponentials of a full (unmasked) block against reference -mneg: y = s * cs - m for a
      // pair of columns in one f32x2 FMA; kPolyPairsOf8 of every 8 pairs take the FMA-pipe
      // exponential, the rest the special-function unit; the row sum is kept in two f32x2
      // accumulators.  Returns the row sum of the block.
      auto exp_full = [&](float mneg) -> float {
        const uint64_t cs2 = f2_pack(cs, cs), mn2 = f2_pack(mneg, mneg);
        uint64_t sa = f2_pack(0.f, 0.f), sb2 = f2_pack(0.f, 0.f);
        float q0p = 0.f, q1p = 0.f;  // FP8: the previous pair, packed with the next one
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const uint64_t y = f2_fma(f2_pack(x[c], x[c + 1]), cs2, mn2);
          float p0, p1;
          if (((c >> 1) & 7) < kPolyPairsOf8) {
            ex2_poly2(y, p0, p1);
          } else {
            float y0, y1;
            f2_unpack(y, y0, y1);
            p0 = ex2(y0);
            p1 = ex2(y1);
          }
          if ((c >> 1) & 1)
            sb2 = f2_add(sb2, f2_pack(p0, p1));
          else
            sa = f2_add(sa, f2_pack(p0, p1));
          if constexpr (FP8) {
            if ((c >> 1) & 1)
              put_word(c >> 2, pack_e4m3x4(q0p, q1p, p0, p1));
            else
              q0p = p0, q1p = p1;
          } else {
            put_word(c >> 1, pack_bf16(p0, p1));
          }
        }
        float s0, s1, s2, s3;
        f2_unpack(sa, s0, s1);
        f2_unpack(sb2, s2, s3);
        return (s0 + s1) + (s2 + s3);
      };
      // Row max with 3-input max (two new columns per instruction, four chains), scaled.
      auto block_max = [&]() -> float {
        float mx0 = fmaxf(x[0], x[1]), mx1 = fmaxf(x[2], x[3]), mx2 = fmaxf(x[4], x[5]), mx3 = fmaxf(x[6], x[7]);
#pragma unroll
        for (int c = 8; c < 128; c += 8) {
          mx0 = max3(mx0, x[c], x[c + 1]);
          mx1 = max3(mx1, x[c + 2], x[c + 3]);
          mx2 = max3(mx2, x[c + 4], x[c + 5]);
          mx3 = max3(mx3, x[c + 6], x[c + 7]);
        }
        return max3(mx0, mx1, fmaxf(mx2, mx3)) * cs;
      };

      int lim = 127;  // last visible column of this row in this block
      if (edge) {
        lim = a.N - 1 - 128 * jg;
        if (a.causal) lim = min(lim, qrow - 128 * jg);
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim) x[c] = -INFINITY;
      }
      const float mblk = block_max();
      const bool move = mblk > m_ref + C::MOVE;
      float alpha = 1.f;
      if (move) {
        alpha = ex2(m_ref - mblk);  // 0 when m_ref is still -inf
        m_ref = mblk;
      }
      l *= alpha;
      // P_t V_{j-1} must have been added into O_t before P_t is rewritten or O_t rescaled
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done(t), (np - 1) & 1, wc));
        if (!ok) break;
      }
      float mneg = (m_ref == -INFINITY) ? 0.f : -m_ref;
      if constexpr (FP8) mneg += C::P_SHIFT;
      if (store_pending) {  // the previous item's O store has read this warp's rows of P_t
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
        store_pending = false;
      }
      float rsum;
      if (!edge) {
        rsum = exp_full(mneg);
      } else {
        // the block with the diagonal or the ragged tail: masked columns are exactly 0
        float rs0 = 0.f, rs1 = 0.f;
        if constexpr (FP8) {
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            const float p0 = (c > lim) ? 0.f : ex2(fmaf(x[c], cs, mneg));
            const float p1 = (c + 1 > lim) ? 0.f : ex2(fmaf(x[c + 1], cs, mneg));
            const float p2 = (c + 2 > lim) ? 0.f : ex2(fmaf(x[c + 2], cs, mneg));
            const float p3 = (c + 3 > lim) ? 0.f : ex2(fmaf(x[c + 3], cs, mneg));
            rs0 += p0;
            rs1 += p1;
            rs0 += p2;
            rs1 += p3;
            put_word(c >> 2, pack_e4m3x4(p0, p1, p2, p3));
          }
        } else {
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            const float p0 = (c > lim) ? 0.f : ex2(fmaf(x[c], cs, mneg));
            const float p1 = (c + 1 > lim) ? 0.f : ex2(fmaf(x[c + 1], cs, mneg));
            rs0 += p0;
            rs1 += p1;
            put_word(c >> 1, pack_bf16(p0, p1));
          }
        }
        rsum = rs0 + rs1;
      }
      l += rsum;
      if ((j > 0 || carry) && __any_sync(0xffffffffu, move)) {
        // O_t holds sum_{j' < j} of P V (and a carried output) relative to the old reference:
        // rescale by alpha.
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t o[32];
          tmem_ld32(tOrow + cc, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tOrow + cc, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full(t));
      ++np;
    }

    if (ok) {
      // ---------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(o_full(t), no & 1, wc));
      ++no;
      if (ok) {
        tc_fence_after();
        const float inv = (l > 0.f) ? vmul / l : 0.f;
        const int row0 = wk.q0 + 128 * t + 32 * wq;
        if (!PARTIAL) {
          // P_t is dead once o_full has fired; each warp stages and stores its own 32 rows, the
          // rows whose P it writes, OST_BOXES 64-column boxes per pass (FP8: two passes, the
          // second after the first store has read the staging)
          uint8_t* stage = gb + C::OST_OFF + t * C::OST_STRIDE;
#pragma unroll
          for (int b0 = 0; b0 < D / 64; b0 += C::OST_BOXES) {
            if (b0 > 0) {
              if (lane == 0) bulk_wait_read0();
              __syncwarp();
            }
#pragma unroll
            for (int bb = 0; bb < C::OST_BOXES && b0 + bb < D / 64; ++bb) {
              const int b = b0 + bb;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                uint32_t o[32];
                tmem_ld32(tOrow + 64 * b + 32 * h, o);
                tmem_wait_ld();
                reg_fence(o);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                  uint4 v;
                  v.x = pack_bf16(__uint_as_float(o[8 * cc + 0]) * inv, __uint_as_float(o[8 * cc + 1]) * inv);
                  v.y = pack_bf16(__uint_as_float(o[8 * cc + 2]) * inv, __uint_as_float(o[8 * cc + 3]) * inv);
                  v.z = pack_bf16(__uint_as_float(o[8 * cc + 4]) * inv, __uint_as_float(o[8 * cc + 5]) * inv);
                  v.w = pack_bf16(__uint_as_float(o[8 * cc + 6]) * inv, __uint_as_float(o[8 * cc + 7]) * inv);
                  const int chunk = h * 4 + cc;  // 16-byte chunk within the 128-byte row
                  *reinterpret_cast<uint4*>(stage + bb * 16384 + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
                }
              }
            }
            if (b0 + C::OST_BOXES >= D / 64) {
              tc_fence_before();
              mbar_arrive(o_free(t));  // O_t is read: the next item's first P V may overwrite it
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && row0 < a.N) {
              for (int bb = 0; bb < C::OST_BOXES && b0 + bb < D / 64; ++bb)
                tma_store_3d(&tmO, sb + C::OST_OFF + t * C::OST_STRIDE + bb * 16384 + wq * 4096, 64 * (b0 + bb),
                             row0, bh);
              bulk_commit();
            }
            __syncwarp();
          }
          store_pending = true;  // waited for before this warp next writes P_t, or at exit
          if (qrow < a.N)
            a.lse[(size_t)bh * a.N + qrow] =
                (l > 0.f) ? (m_ref - C::P_SHIFT + log2f(l)) * 0.69314718055994530942f : -INFINITY;
        } else {
          // fp32 partial O_s = O / l of this split, staged in the (now idle) K/V ring and P tiles as
          // 32-column, 128-byte-swizzled boxes and written by TMA; then LSE_s.
          constexpr int PBOX = D / 32;
          const uint32_t pstage = C::KV_OFF + t * (128 * D * 4);
          uint8_t* stage = gb + pstage;
#pragma unroll
          for (int b = 0; b < PBOX; ++b) {
            uint32_t o[32];
            tmem_ld32(tOrow + 32 * b, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              float4 v = make_float4(__uint_as_float(o[4 * cc + 0]) * inv, __uint_as_float(o[4 * cc + 1]) * inv,
                                     __uint_as_float(o[4 * cc + 2]) * inv, __uint_as_float(o[4 * cc + 3]) * inv);
              *reinterpret_cast<float4*>(stage + b * 16384 + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
            }
          }
          tc_fence_before();
          mbar_arrive(o_free(t));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < a.N) {
            for (int b = 0; b < PBOX; ++b)
              tma_store_3d(&tmO, sb + pstage + b * 16384 + wq * 4096, 32 * b, row0, split * a.BH + bh);
            bulk_commit();
            bulk_wait_read0();
          }
          __syncwarp();
          if (qrow < a.N)
            a.lse[((size_t)split * a.BH + bh) * a.N + qrow] =
                (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994530942f : -INFINITY;
        }
      }
    }
    }  // items
    if (lane == 0) bulk_wait0();  // every O store has completed before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, C::TMEM_COLS);
  }
}

template <int D, bool PARTIAL, bool FP8 = false>
static cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& to, const FwdArgs& a, cudaStream_t stream) {
  using C = FwdCfg<D, FP8>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  static_assert(C::SMEM > 116 * 1024, "one CTA per SM: each allocates all 512 TMEM columns");
  static_assert(2 * 128 * D * 4 <= C::NS * C::TILE + 2 * C::PTILE, "partial-output staging must fit the ring and P");
  static_assert(C::OST_BOXES >= 1 && C::OST_BOXES * 16384 <= C::OST_STRIDE &&
                    C::OST_OFF + 2 * C::OST_STRIDE <= C::BAR_OFF,
                "output staging must fit");
  static bool attr_set[64];  // per device: the attribute outlives the call
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(fa_fwd_kernel<D, PARTIAL, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const long long items = (long long)a.BH * a.nqb * a.nsplit;
  if (items > INT_MAX) return cudaErrorInvalidValue;
  FwdArgs b = a;
  long long grid = items;
  b.persistent = 0;
  if (!PARTIAL) {
    // The whole key range (bf16 or FP8): at most one CTA per SM, each walking its pairs of items,
    // when the items are of equal length (no mask) or many per SM.  Under the causal mask with
    // few items per SM the hardware's dispatch of one CTA per item (to whichever SM frees up
    // first) balances the uneven items better.  Measured on B200: persistent is 1-3 % faster
    // at B=1 H=32 N=16384 causal (13.8 items per SM) and 6 % at B=4 H=16 N=1024 without mask,
    // 17 % slower at B=2 H=16 N=4096 causal (3.5 items per SM).
    static int sms[64];
    if (dev >= 0 && dev < 64 && sms[dev] == 0) {
      e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
    }
    const long long nsm = (dev >= 0 && dev < 64 && sms[dev] > 0) ? sms[dev] : 148;
    if (!a.causal || items >= 8 * nsm) {
      b.persistent = 1;
      grid = std::min((items + 1) / 2, nsm);
    }
  }
  FA_DBG(b.visits = debug_visits(0); b.visits_cap = kDebugVisitInts;)
  fa_fwd_kernel<D, PARTIAL, FP8><<<(unsigned)grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, to, b);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdArgs& a, cudaStream_t stream) {
  if (a.nsplit > 1) {
    if (d == 64) return launch_fwd_t<64, true>(tq, tk, tv, to, a, stream);
    return launch_fwd_t<128, true>(tq, tk, tv, to, a, stream);
  }
  if (d == 64) return launch_fwd_t<64, false>(tq, tk, tv, to, a, stream);
  return launch_fwd_t<128, false>(tq, tk, tv, to, a, stream);
}

cudaError_t launch_fwd_partial(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& to, const FwdArgs& a, cudaStream_t stream) {
  if (d == 64) return launch_fwd_t<64, true>(tq, tk, tv, to, a, stream);
  return launch_fwd_t<128, true>(tq, tk, tv, to, a, stream);
}

cudaError_t launch_fwd_fp8(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const FwdArgs& a, cudaStream_t stream) {
  if (d != 128 || a.nsplit != 1) return cudaErrorNotSupported;
  return launch_fwd_t<128, false, true>(tq, tk, tv, to, a, stream);
}

// Combines the split-wise partial results of one query row, using the two-block softmax merge
// of "Flash Attention" (special-jiahao.github.io), section 增量求解 softmax, applied to nsplit
// blocks: with M = max_s LSE_s and weights w_s = e^{LSE_s - M} (each block's sum rescaled to
// the common max), O = sum_s w_s O_s / sum_s w_s and LSE = M + ln sum_s w_s.  Splits with
// LSE_s = -inf hold no visible key and contribute nothing; their partial rows are never
// written.  One warp per row; lane holds D/32 columns.  S > 0: exactly S splits, with every
// load of the row issued before any is used (the empty splits' rows are read, inside the
// workspace, and their terms dropped by a select, so stale values never reach the sum);
// S = 0: any number of splits, the empty ones skipped by a branch.
template <int D, int S>
__global__ void __launch_bounds__(256) fa_fwd_merge_kernel(const float* __restrict__ o_part,
                                                           const float* __restrict__ lse_part,
                                                           __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                                           int nsplit, long long rows) {
  constexpr int V = D / 32;
  const int lane = threadIdx.x & 31;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  if constexpr (S > 0) {
    for (long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows; row += nw) {
      float L[S];
      float x[S][V];
#pragma unroll
      for (int sp = 0; sp < S; ++sp) L[sp] = lse_part[sp * rows + row];
#pragma unroll
      for (int sp = 0; sp < S; ++sp) {
        const float* src = o_part + ((size_t)sp * rows + row) * D + lane * V;
        if (V == 4) {
          const float4 t = *reinterpret_cast<const float4*>(src);
          x[sp][0] = t.x, x[sp][1] = t.y, x[sp][2 % V] = t.z, x[sp][3 % V] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(src);
          x[sp][0] = t.x, x[sp][1] = t.y;
        }
      }
      float m = L[0];
#pragma unroll
      for (int sp = 1; sp < S; ++sp) m = fmaxf(m, L[sp]);
      float acc[V];
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] = 0.f;
      float wsum = 0.f;
#pragma unroll
      for (int sp = 0; sp < S; ++sp) {
        const bool live = (L[sp] != -INFINITY);
        const float w = live ? expf(L[sp] - m) : 0.f;
        wsum += w;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = live ? fmaf(w, x[sp][e], acc[e]) : acc[e];
      }
      const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
      __nv_bfloat16* dst = o + (size_t)row * D + lane * V;
      if (V == 4) {
        uint2 u;
        u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
        u.y = pack_bf16(acc[2 % V] * inv, acc[3 % V] * inv);
        *reinterpret_cast<uint2*>(dst) = u;
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0] * inv, acc[1] * inv);
      }
      if (lane == 0) lse[row] = (wsum > 0.f) ? m + logf(wsum) : -INFINITY;
    }
  } else {
    for (long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows; row += nw) {
      float m = -INFINITY;
      for (int sp = 0; sp < nsplit; ++sp) m = fmaxf(m, lse_part[sp * rows + row]);
      float acc[V];
  #pragma unroll
      for (int e = 0; e < V; ++e) acc[e] = 0.f;
      float wsum = 0.f;
      if (m != -INFINITY) {
        for (int sp = 0; sp < nsplit; ++sp) {
          const float L = lse_part[sp * rows + row];
          if (L == -INFINITY) continue;
          const float w = expf(L - m);
          wsum += w;
          const float* src = o_part + ((size_t)sp * rows + row) * D + lane * V;
          if (V == 4) {
            const float4 x = *reinterpret_cast<const float4*>(src);
            acc[0] += w * x.x; acc[1] += w * x.y; acc[2] += w * x.z; acc[3] += w * x.w;
          } else {
            const float2 x = *reinterpret_cast<const float2*>(src);
            acc[0] += w * x.x; acc[1] += w * x.y;
          }
        }
      }
      const float inv = (wsum > 0.f) ? 1.f / wsum : 0.f;
      __nv_bfloat16* dst = o + (size_t)row * D + lane * V;
      if (V == 4) {
        uint2 u;
        u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
        u.y = pack_bf16(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(dst) = u;
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0] * inv, acc[1] * inv);
      }
      if (lane == 0) lse[row] = (wsum > 0.f) ? m + logf(wsum) : -INFINITY;
    }
  }
}

cudaError_t launch_fwd_merge(const float* o_part, const float* lse_part, void* o, float* lse, int nsplit,
                             long long rows, int d, cudaStream_t stream) {
  long long blocks = (rows + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  if (blocks < 1) blocks = 1;
  auto* out = reinterpret_cast<__nv_bfloat16*>(o);
  const unsigned g = (unsigned)blocks;
#define FA_MERGE(DD, SS) fa_fwd_merge_kernel<DD, SS><<<g, 256, 0, stream>>>(o_part, lse_part, out, lse, nsplit, rows)
  if (d == 64) {
    switch (nsplit) {
      case 2: FA_MERGE(64, 2); break;
      case 3: FA_MERGE(64, 3); break;
      case 4: FA_MERGE(64, 4); break;
      default: FA_MERGE(64, 0);
    }
  } else {
    switch (nsplit) {
      case 2: FA_MERGE(128, 2); break;
      case 3: FA_MERGE(128, 3); break;
      case 4: FA_MERGE(128, 4); break;
      default: FA_MERGE(128, 0);
    }
  }
#undef FA_MERGE
  return cudaGetLastError();
}

}  // namespace fa
