// Backward attention kernels for sm_100a (placeholder until the kernels land).
#include "fa_internal.h"

namespace fa {

size_t bwd_workspace_bytes(const AttnShape& s) {
  const size_t rows = static_cast<size_t>(s.B) * s.Hq * s.N;
  return rows * 4 + rows * s.d * 4 + 256;
}

cudaError_t launch_bwd(const AttnShape&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                       const CUtensorMap&, const void*, const void*, const float*, void*, void*, void*, void*,
                       const LaunchCtl&, cudaStream_t) {
  return cudaErrorNotYetImplemented;
}

}  // namespace fa
