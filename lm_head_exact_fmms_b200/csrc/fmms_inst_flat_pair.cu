// fmms_inst_flat_pair.cu -- the fused kernel in flat mode on CTA pairs, built for every batch tile.
#include "fmms_kernel.cuh"
#include "launch.h"

namespace fmms {

cudaError_t launch_flat_pair(int BN, const CUtensorMap &tw, const PartMaps &twp,
                           const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream) {
  switch (BN) {
#define FMMS_CASE(n) \
  case n: return launch_pair_t<n, kModeFlat>(tw, twp, th, p, stream);
    FMMS_FOR_EACH_BN(FMMS_CASE)
#undef FMMS_CASE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t pair_units_flat(int BN, int *units) {
  switch (BN) {
#define FMMS_CASE(n) \
  case n: return pair_units_t<n, kModeFlat>(units);
    FMMS_FOR_EACH_BN(FMMS_CASE)
#undef FMMS_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fmms
