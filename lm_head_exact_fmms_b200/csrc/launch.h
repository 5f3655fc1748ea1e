// launch.h -- host-side launchers of the FMMS kernels (internal to libfmms).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fmms_common.cuh"

namespace fmms {

// Tensor maps of W for partial tiles: boxes of 8, 16, 32 and 64 rows.  A
// partial tile of 8k rows is loaded as at most four boxes, one for each
// binary digit of k, instead of k boxes of 8 rows.
struct PartMaps {
  CUtensorMap box[4];
};

// Batch tile (MMA N) of a launch of `rows` rows: the next multiple of 16,
// at most 256.
int fmms_batch_tile(int rows);

// Per-mode launchers for every batch tile (fmms_inst_*.cu).
cudaError_t launch_flat(int BN, bool merge, const CUtensorMap &tw, const PartMaps &twp,
                        const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream);
cudaError_t launch_grouped(int BN, bool merge, const CUtensorMap &tw, const PartMaps &twp,
                           const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream);
cudaError_t launch_logits(int BN, bool merge, const CUtensorMap &tw, const PartMaps &twp,
                          const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream);
cudaError_t launch_flat_pair(int BN, const CUtensorMap &tw, const PartMaps &twp,
                             const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream);
cudaError_t launch_grouped_pair(int BN, const CUtensorMap &tw, const PartMaps &twp,
                                const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream);
cudaError_t pair_units_flat(int BN, int *units);
cudaError_t pair_units_grouped(int BN, int *units);

// The fused kernel in mode kModeFlat / kModeGrouped / kModeLogits with batch
// tile BN, grid p.num_ctas x kThreads threads.
cudaError_t launch_fmms(int mode, int BN, bool merge, const CUtensorMap &tw, const PartMaps &twp,
                        const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream);

// The flat or grouped kernel on CTA pairs (clusters of two, tcgen05
// cta_group::2): p.num_ctas CTAs (even), th with boxes of BN/2 rows.
cudaError_t launch_fmms_pair(int mode, int BN, const CUtensorMap &tw, const PartMaps &twp,
                             const CUtensorMap &th, const FmmsParams &p, cudaStream_t stream);

// How many CTA pairs of the BN pair kernel of `mode` can be resident at once.
cudaError_t fmms_pair_units(int mode, int BN, int *units);

// Group-Gumbel-Max merge of the grouped partials of one launch (B rows).
struct MergeParams {
  GroupPartial *partials;        // [slots][B]; zeroed as they are read
  unsigned long long *gkeys;     // [G][B] published maxima to re-zero, or null
  int B, b_off, V, G, num_ctas, ngran;
  int pair;                      // 1: partials of a CTA-pair launch (two slots per segment)
  uint64_t seed;
  const uint64_t *row_seeds;
  uint32_t step;
  int32_t *out_idx;              // [B], offset to this launch
  void *summary;                 // fs_group_summary [B][G] offset to this launch, or null
  // Debug-build bounds checks (entries): the status word, the partial records
  // and published maxima in the workspace, rows of row_seeds.
  int *err;
  long long partials_cap, gkeys_cap;
  int rows_total;
};
cudaError_t launch_group_merge(const MergeParams &m, cudaStream_t stream);

// Second kernel of the unfused mode: samples from fp32 logits [B][V].
struct SampleLogitsParams {
  const float *logits;           // [B][V], offset to this launch
  int B, b_off, V;
  float inv_temp;
  uint64_t seed;
  const uint64_t *row_seeds;
  uint32_t step;
  const uint32_t *mask;
  int mask_words;
  unsigned long long *keys;      // workspace [B]
  unsigned int *ticket;
  int32_t *out_idx;
  int num_sms;
  int *err;                      // status word (debug-build bounds checks)
  int rows_total;                // rows of row_seeds and mask (the whole call)
};
cudaError_t launch_sample_logits(const SampleLogitsParams &s, cudaStream_t stream);

// Top-k sampling over the fp32 logits: two launches (per-block candidate
// lists by radix histograms, then one block per row selects and samples).
// `scratch` holds topk_scratch_bytes(s.B, s.V, K, s.num_sms) bytes; no
// contents carry over between calls.
size_t topk_scratch_bytes(int rows, int V, int K, int num_sms);
cudaError_t launch_topk_sample(const SampleLogitsParams &s, int K, void *scratch,
                               cudaStream_t stream);

// Group-Gumbel-Max over per-group summaries [G][B] (fs_group_summary records).
cudaError_t launch_merge_summaries(const void *summaries, int G, int B, uint64_t seed,
                                   const uint64_t *row_seeds, uint32_t step, int32_t *out_idx,
                                   cudaStream_t stream);

// Waits, at most timeout_us, for call `seq` of this rank's exchange area and
// copies its tokens (or writes -1 and marks the call failed).
cudaError_t launch_tp_wait(TpArea *area, int B, uint32_t seq, int32_t *out_idx,
                           uint32_t timeout_us, cudaStream_t stream);

// The two-kernel reduction: decodes the fused kernel's published keys
// [sample][kMaxBN rows] of this launch's B rows into tokens (or, with
// out_keys, packed keys XOR 2^63) and re-zeroes them for the next call.
cudaError_t launch_decode_published(unsigned long long *keys, int B, int num_samples,
                                    int32_t *out_idx, long long *out_keys, int *err,
                                    int keys_cap, cudaStream_t stream);

// Decodes packed keys (XOR 2^63, as fs_sample_shard_keys writes them) to tokens.
cudaError_t launch_keys_to_tokens(const long long *keys, int B, int32_t *out_idx,
                                  cudaStream_t stream);

cudaError_t launch_philox_test(const uint32_t *ctr, const uint32_t *key, uint32_t *out, int64_t n,
                               cudaStream_t stream);
cudaError_t launch_gumbel_test(const uint32_t *r, float *g, int64_t n, cudaStream_t stream);

}  // namespace fmms
