// fmms_inst_logits.cu -- the fused kernel in logits mode (the unfused measurement path), built for every batch tile.
#include "fmms_kernel.cuh"
#include "launch.h"

namespace fmms {

cudaError_t launch_logits(int BN, bool merge, const CUtensorMap &tw, const PartMaps &twp,
                          const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream) {
  switch (BN) {
#define FMMS_CASE(n) \
  case n:                                                                 \
    return merge ? launch_t<n, kModeLogits, (n <= 64)>(tw, twp, th, p, stream)     \
                 : launch_t<n, kModeLogits, false>(tw, twp, th, p, stream);
    FMMS_FOR_EACH_BN(FMMS_CASE)
#undef FMMS_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fmms
