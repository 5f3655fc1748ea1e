// fmms_kernel.cu -- dispatch of the fused matmul-sample kernel by mode, batch
// tile and CTA arrangement.  The kernel itself is in fmms_kernel.cuh; each
// fmms_inst_*.cu builds one mode for every batch tile, so that the
// instantiations compile in parallel.
#include "launch.h"

namespace fmms {

cudaError_t launch_fmms(int mode, int BN, bool merge, const CUtensorMap &tw, const PartMaps &twp,
                        const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream) {
  switch (mode) {
    case kModeFlat: return launch_flat(BN, merge, tw, twp, th, p, stream);
    case kModeGrouped: return launch_grouped(BN, merge, tw, twp, th, p, stream);
    case kModeLogits: return launch_logits(BN, merge, tw, twp, th, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fmms_pair(int mode, int BN, const CUtensorMap &tw, const PartMaps &twp,
                             const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream) {
  switch (mode) {
    case kModeFlat: return launch_flat_pair(BN, tw, twp, th, p, stream);
    case kModeGrouped: return launch_grouped_pair(BN, tw, twp, th, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t fmms_pair_units(int mode, int BN, int *units) {
  switch (mode) {
    case kModeFlat: return pair_units_flat(BN, units);
    case kModeGrouped: return pair_units_grouped(BN, units);
    default: return cudaErrorInvalidValue;
  }
}

int fmms_batch_tile(int rows) {
  const int bn = (rows + 15) / 16 * 16;
  return bn < 16 ? 16 : (bn > kMaxBN ? kMaxBN : bn);
}

}  // namespace fmms
