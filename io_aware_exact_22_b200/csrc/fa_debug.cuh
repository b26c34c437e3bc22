// fa_debug.cuh - device-side checks of the debug build (libfa_debug.so, compiled with
// FA_DEBUG).  In the release build every FA_DBG(...) statement compiles to nothing.
//
// Visit log: each kernel counts, per (batch * head, query tile, key tile), how many times it
// processed that tile pair, in a [BH][nq][nk] block of int counters (one block per kernel kind,
// see debug_visits in fa_internal.cuh); a test compares the counts with the pairs that the
// mask makes visible, exactly.  Index checks: a computed tile index or global offset outside
// its range sets FA_DEV_BOUNDS in the device status word and the access is skipped; nothing
// traps, so the context stays usable and the host reads the bit with fa_get_device_status.
#pragma once

#include "sm100_ptx.cuh"

namespace fa {

#ifdef FA_DEBUG
#define FA_DBG(...) __VA_ARGS__
// One visit of tile pair (qt, kt) of head bh in a [BH][nq][nk] block of `cap` counters.
__device__ __forceinline__ void dbg_visit(int* v, long long cap, uint32_t* status, int bh, int nq, int qt,
                                          int nk, int kt) {
  if (v == nullptr) return;
  const long long idx = ((long long)bh * nq + qt) * nk + kt;
  if (qt < 0 || qt >= nq || kt < 0 || kt >= nk || bh < 0 || idx < 0 || idx >= cap) {
    atomicOr(status, FA_DEV_BOUNDS);
    return;
  }
  atomicAdd(v + idx, 1);
}
// True when `ok` holds; otherwise records FA_DEV_BOUNDS and returns false.
__device__ __forceinline__ bool dbg_check(bool ok, uint32_t* status) {
  if (!ok) atomicOr(status, FA_DEV_BOUNDS);
  return ok;
}
#else
#define FA_DBG(...)
#endif

}  // namespace fa
