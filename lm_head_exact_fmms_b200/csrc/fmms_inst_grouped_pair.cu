// fmms_inst_grouped_pair.cu -- the fused kernel in grouped mode on CTA pairs, built for every batch tile.
#include "fmms_kernel.cuh"
#include "launch.h"

namespace fmms {

cudaError_t launch_grouped_pair(int BN, const CUtensorMap &tw, const PartMaps &twp,
                           const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream) {
  switch (BN) {
#define FMMS_CASE(n) \
  case n: return launch_pair_t<n, kModeGrouped>(tw, twp, th, p, stream);
    FMMS_FOR_EACH_BN(FMMS_CASE)
#undef FMMS_CASE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t pair_units_grouped(int BN, int *units) {
  switch (BN) {
#define FMMS_CASE(n) \
  case n: return pair_units_t<n, kModeGrouped>(units);
    FMMS_FOR_EACH_BN(FMMS_CASE)
#undef FMMS_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fmms
