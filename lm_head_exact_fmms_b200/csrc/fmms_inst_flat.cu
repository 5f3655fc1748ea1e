// fmms_inst_flat.cu -- the fused kernel in flat mode on single CTAs, built for every batch tile
// (up to 64 rows also with merged 8-row partial tiles).
#include "fmms_kernel.cuh"
#include "launch.h"

namespace fmms {

cudaError_t launch_flat(int BN, bool merge, const CUtensorMap &tw, const PartMaps &twp,
                        const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream) {
  switch (BN) {
#define FMMS_CASE(n) \
  case n:                                                                 \
    return merge ? launch_t<n, kModeFlat, (n <= 64)>(tw, twp, th, p, stream)     \
                 : launch_t<n, kModeFlat, false>(tw, twp, th, p, stream);
    FMMS_FOR_EACH_BN(FMMS_CASE)
#undef FMMS_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fmms
