// fa_internal.cuh - declarations shared by the host side of libfa.so (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace fa {

struct FwdArgs {
  uint32_t* status;  // device status word
  float* lse;        // [BH, N] fp32; with key splits: [nsplit, BH, N] partial LSEs
  int N;             // sequence length
  int BH;            // batch * heads
  int nqb;           // query blocks of 256 rows per head
  int causal;        // 0 / 1
  float scale_log2;  // scale * log2(e)
  int nsplit;        // key-range splits per (head, query block); 1 = whole key range
  int group = 1;      // work order: heads per group, heaviest query block first within a group
  int persistent = 0;  // set by the launcher: CTAs walk the work list in pairs (see fa_fwd_kernel)
  // FP8 forward only: per-(b,h) dequantisation factors [BH], or null for 1
  const float* descale_q = nullptr;
  const float* descale_k = nullptr;
  const float* descale_v = nullptr;
  // Carried partial result (bf16 kernels, whole key range): when set, the rows continue from
  // a normalised output carry_o [BH, N, d] fp32 and its natural-log LSE carry_lse [BH, N] over
  // other keys (rows with LSE = -inf have seen none)
  const float* carry_o = nullptr;
  const float* carry_lse = nullptr;
  // debug build: visit counters [BH][ceil(N/128)][ceil(N/128)] (null in the release build)
  int* visits = nullptr;
  long long visits_cap = 0;
};

struct BwdArgs {
  uint32_t* status;  // device status word
  const float* lse;  // [BH, N] fp32, natural log
  const float* ld;   // [BH, ceil(N/64), 128] fp32: per 64-row query tile, 64 x LSE*log2(e)
                     // then 64 x D_i = rowsum(dO o O); rows past N hold +inf and 0
  float* dq_acc;     // [BH, N, d] fp32 accumulator (zeroed by the pre-kernel)
  int N;
  int BH;
  int causal;
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  // When set (d = 128, with the dQ path): scale * dK and dV of this call are added into these
  // fp32 [BH, N, d] accumulators instead of being stored as bf16 (the sequence-sharded backward)
  float* dk_acc = nullptr;
  float* dv_acc = nullptr;
  int acc_overwrite = 0;  // with dk_acc: store into the accumulators instead of adding
  int group = 1;  // work order: heads per group, heaviest key tile first within a group
  // two ints in device memory, zero before each launch of the key-tile kernel (the pre-kernel
  // zeroes them; the kernel's last CTA zeroes them again on exit): the next unclaimed item
  // and the number of CTAs done
  int* work = nullptr;
  // debug build: visit counters of the kernel launched with these arguments (null in release)
  int* visits = nullptr;
  long long visits_cap = 0;
};

// Debug build: device address of the visit-counter block of one kernel kind (0 forward,
// 1 backward key-tile kernel, 2 deterministic dQ kernel), kDebugVisitInts counters each;
// nullptr in the release build.
constexpr long long kDebugVisitInts = 1LL << 20;
int* debug_visits(int kind);

// Backward dQ accumulation: of each 64-row query tile, the first kBwdDqRedRows rows are added
// into the fp32 accumulator with per-thread reductions, the rest with one TMA reduce-add
// (tensor-map box of 64 - kBwdDqRedRows rows).  Measured at B=2 H=16 N=4096, B=1 H=32
// N=16384 (causal) and B=4 H=16 N=4096 (non-causal): 0 (every row by TMA) is 0.5-1.8 %
// faster than 32, and 48 is 2.5-3 % slower.
constexpr int kBwdDqRedRows = 0;

// Device address of this library's status word on the current device (nullptr on error).
uint32_t* device_status_word();

// Launches the bounded-wait self-test kernel (see fa_selftest_wait_timeout).
cudaError_t launch_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);

// Tensor maps for a bf16 [BH, N, d] tensor, 128-byte swizzle, box = 64 columns x `rows`
// (make_*: served from a cache of encoded maps; encode_*: always encodes).
// 3-D map over an E4M3 tensor [BH, N, d] (one byte per element), box {128, box_rows},
// 128-byte swizzle.
bool make_tmap_e4m3(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_rows);
bool make_tmap_bf16(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_rows);
bool encode_tmap_bf16(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_rows);
bool encode_tmap_f32(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_inner, int box_rows,
                     bool swizzle128);

// With a.nsplit == 1, `to` maps the bf16 output; with a.nsplit > 1 it maps the fp32 partial
// outputs [nsplit * BH, N, d] (box 32 x 32, 128-byte swizzle) and a.lse the partial LSEs.
cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdArgs& a, cudaStream_t stream);
// Partial outputs (fp32 O / l and LSE) for a.nsplit >= 1 key ranges, whatever a.nsplit is; `to`
// maps the fp32 partials [a.nsplit * BH, N, d].
cudaError_t launch_fwd_partial(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& to, const FwdArgs& a, cudaStream_t stream);
// FP8 (E4M3) inputs, d = 128, whole key range; Q/K/V maps from make_tmap_e4m3 (128-row boxes)
cudaError_t launch_fwd_fp8(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const FwdArgs& a, cudaStream_t stream);
// Combines nsplit partial (O_s, LSE_s) into bf16 O and fp32 LSE.
cudaError_t launch_fwd_merge(const float* o_part, const float* lse_part, void* o, float* lse, int nsplit,
                             long long rows, int d, cudaStream_t stream);

cudaError_t launch_bwd_pre(const void* o, const void* dO, const float* lse, float* ld, float* dq_acc, int* work,
                           int BH, int N, int d, cudaStream_t stream);
// fp32 [BH, N, d] tensor map without swizzle, box = box_inner columns x box_rows rows.
bool make_tmap_f32(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_inner, int box_rows,
                   bool swizzle128 = false);

// with_dq = false: dK and dV only (no dQ accumulation; tdq and a.dq_acc unused).
cudaError_t launch_bwd_main(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const CUtensorMap& tdo,
                            const CUtensorMap& tdk, const CUtensorMap& tdv,
                            const CUtensorMap& tdq, const BwdArgs& a, cudaStream_t stream,
                            bool with_dq = true);
// Deterministic dQ (query-tile-outer, accumulated in TMEM, written once): tq/tdo with 128-row
// boxes, tk/tv with 64-row boxes, tdq the bf16 dQ with 32-row boxes; needs a.ld filled.
cudaError_t launch_bwd_dq(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a,
                          cudaStream_t stream);
// acc += x over elems fp32 values (a multiple of 4, 16-byte aligned).
cudaError_t launch_acc_add(float* acc, const float* x, long long elems, cudaStream_t stream);
cudaError_t launch_bwd_post(const float* dq_acc, void* dq, long long elems, float scale,
                            cudaStream_t stream);

}  // namespace fa
