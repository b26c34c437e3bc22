// fa_bwd.cu - backward of exact attention (recomputation; "xinc.fun archive 235", section 7).
#include "fa_internal.cuh"
#include "sm100_ptx.cuh"

namespace fa {

cudaError_t launch_bwd_pre(const void*, const void*, float*, float*, long long, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_bwd_main(int, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                            const BwdArgs&, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_bwd_post(const float*, void*, long long, float, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace fa
