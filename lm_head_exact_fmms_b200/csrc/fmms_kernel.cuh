// fmms_kernel.cuh -- the fused matmul-sample (FMMS) kernel for sm_100a (templates;
// fmms_kernel.cu dispatches, fmms_inst_*.cu instantiate one mode each).
//
// What it computes (FlashSampling, arXiv:2603.15854, abstract): logits of a
// vocabulary tile are formed on chip, scaled by 1/T, masked, perturbed with
// Gumbel noise, and only one (score, token) maximiser per row and tile
// survives; a reduction over tiles gives one token per row.  The B x V
// logits never reach HBM (except in the logits mode kept for measurement).
//
// How (B200 design; the Triton kernel the pages describe is prior art only):
//  * one persistent CTA per SM; each CTA owns a contiguous, 8-row-granular
//    slice of the vocabulary (split-V), so small batches still keep all 148
//    SMs streaming W and no W row is read twice;
//  * swap-AB MMA: A = 128 vocabulary rows of W (M = 128), B = the batch of
//    hidden states (N = the batch tile, a multiple of 16 up to 256), D = a
//    128-lane x N-column fp32 accumulator in tensor memory; the tile's
//    vocabulary rows land on TMEM lanes, i.e. on epilogue threads;
//  * CTA pairs (PAIR): two CTAs of a cluster share one M = 256 MMA
//    (tcgen05 cta_group::2); each stages its own 128 W rows and half of the
//    H rows and drains its own 128 accumulator rows;
//  * warp roles: warp 0 issues TMA loads of W (evict-first) and H
//    (evict-last) into a ring of 3-10 stages of 1-4 64-wide K sub-blocks
//    (128-byte swizzle); warp 1 allocates TMEM and issues tcgen05.mma;
//    warps 2-17 (four per TMEM lane quarter) drain up to four accumulators
//    while the next tiles are being multiplied;
//  * epilogue per 16-column chunk: x = acc / T, Philox4x32-10 noise words for
//    (seed, step, row, token) (one Philox call serves four consecutive
//    tokens; four lanes exchange words with a 4x4 shuffle transpose), a
//    log-free upper bound of each Gumbel value, and only where a bound
//    reaches the row's best published score the exact transform, s = x + g
//    and a 32-lane "transpose-reduce" that leaves each lane pair with the
//    packed max of one column;
//  * flat mode: every improvement of a row's maximum is published with one
//    atomicMax of a packed (score, token) key; the last CTA to finish (atomic
//    ticket, no waiting) decodes the tokens and re-zeroes the keys;
//  * a CTA range's 8-row partial tile either runs as a tile of its own or
//    (MERGE variant) rides along with the first whole tile: its rows get a
//    1 KB slot per stage and a second MMA into an accumulator of its own,
//    sharing the H loads;
//  * grouped mode: per (segment, row) partial (max key, lse pieces) for the
//    Group-Gumbel-Max merge kernel;
//  * logits mode: raw fp32 logits to HBM for the unfused measurement path.
// Every wait is bounded; a CTA that gives up records FS_ERR_DEVICE_TIMEOUT.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fmms_common.cuh"
#include "launch.h"
#include "noise.cuh"
#include "sm100.cuh"

namespace fmms {

// Shared memory a kernel may use beyond the stages: alignment slack,
// barriers and (grouped mode) the combine area.
constexpr int kSmemBudget = 232448 - 1024 - 256;

// K sub-blocks of 64 elements per pipeline stage, and the number of stages.
// Measured on the Qwen3-8B, Qwen3-1.7B and d=8192 heads: what sets the
// streaming rate is the W bytes in flight per SM (stages x sub-blocks x
// 16 KB), with at least three stages so that loads, MMAs and the stage
// hand-back overlap, and at equal bytes the longer per-row bursts of more
// sub-blocks per stage win (fewer handshakes per byte, 128 B more of each W
// row per sub-block).  So: among 1..4 sub-blocks with at least three stages
// (at most ten), the most W bytes in flight, ties to more sub-blocks.
// E.g. single CTAs: 4 x 3 stages at 16 batch rows, 2 x 5 at 32, 3 x 3 at 64.
// CTA pairs at 224 rows and more run tensor-bound, where the MMAs of a stage
// hold it longer and fewer, larger stages pay more: there a choice with one
// sub-block less in flight still counts as a tie (`slack`), so 256 rows take
// 2 x 3 instead of 1 x 7 (measured: B=256 on the Qwen3-8B head 322 -> 305 us,
// on the d=8192 head 504 -> 483 us; 1 x 7 and 3 x 2 both slower).  Below 224
// rows the plain rule measured best (pairs: 3 x 3 at 128 rows, 64 H rows per
// CTA; 2 x 4 at 160 and 192).
constexpr int kMaxStages = 10;
constexpr int stages_for(int ksub, int h_rows, int comb_bytes, int p_bytes) {
  const int fit = (kSmemBudget - comb_bytes) / (ksub * ((kTileM + h_rows) * kBlockK * 2 + p_bytes));
  return fit < kMaxStages ? fit : kMaxStages;
}
constexpr int ksub_for(int h_rows, int comb_bytes, int p_bytes, int slack = 0) {
  int best_bytes = 0;
  for (int k = 1; k <= 4; ++k) {
    const int st = stages_for(k, h_rows, comb_bytes, p_bytes);
    if (st >= 3 && st * k > best_bytes) best_bytes = st * k;
  }
  int best = 1;
  for (int k = 1; k <= 4; ++k) {
    const int st = stages_for(k, h_rows, comb_bytes, p_bytes);
    if (st >= 3 && st * k >= best_bytes - slack) best = k;
  }
  return best;
}

// Tensor-memory columns to allocate: a power of two, at least 32.
constexpr int tmem_cols_for(int cols) {
  int n = 32;
  while (n < cols) n *= 2;
  return n;
}

template <int BN, int MODE, bool PAIR = false, bool MERGE = false>
struct KCfg {
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= kMaxBN, "batch tile: a multiple of 16 rows");
  static_assert(!PAIR || MODE != kModeLogits, "the logits mode runs on single CTAs");
  static constexpr int kHRows = PAIR ? BN / 2 : BN;     // H rows this CTA stages
  static constexpr int kCombBytes = MODE == kModeGrouped ? 4 * BN * 16 : 0;  // grouped only
  // Merged 8-row partial tiles (MERGE; single CTAs of up to 64 batch rows,
  // above that CTA pairs run): each stage starts with one 8-row W slot per
  // sub-block.  The host picks this variant for vocabularies whose split
  // gives many CTAs an 8-row partial tile (the Qwen3 heads: B=1 191.5 ->
  // 186.5 us, B=64 198 -> 192 us); elsewhere the slot only costs ring space
  // (at 16 rows the ring goes from 4 x 3 to 2 x 5 sub-blocks) and the
  // d=8192 head ran 3-4 % slower with it.
  static constexpr bool kMerge = MERGE && !PAIR && BN <= 64;
  static constexpr int kSubP = kMerge ? kGranule * kBlockK * 2 : 0;  // 1 KB per sub-block
  static constexpr int kSub =
      ksub_for(kHRows, kCombBytes, kSubP, PAIR && BN >= 224 ? 1 : 0);  // 64-wide K blocks per stage
  static constexpr int kSubW = kTileM * kBlockK * 2;    // 16 KB of W per sub-block
  static constexpr int kSubH = kHRows * kBlockK * 2;    // this CTA's H rows per sub-block
  static constexpr int kStageP = kSub * kSubP;
  static constexpr int kStageW = kSub * kSubW;
  static constexpr int kStageH = kSub * kSubH;
  static constexpr int kOffW = kStageP;                 // stage layout: [P][W][H]
  static constexpr int kOffH = kStageP + kStageW;
  static constexpr int kStageBytes = kStageP + kStageW + kStageH;
  static constexpr int kStages = stages_for(kSub, kHRows, kCombBytes, kSubP);
  static constexpr int kCW = 16;                        // columns per epilogue chunk
  static constexpr int kChunks = BN / kCW;
  static constexpr int kWarpsPerQuarter = kNumEpiWarps / 4;
  static constexpr int kChunksPerWarp = (kChunks + kWarpsPerQuarter - 1) / kWarpsPerQuarter;
  static constexpr int kAccBufs = 512 / BN < 4 ? 512 / BN : 4;  // accumulators in flight
  static constexpr int kTmemCols = tmem_cols_for(kAccBufs * BN);
  static constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(PAIR ? 2 * kTileM : kTileM, BN);
  static constexpr int kEpiArrivals = PAIR ? 2 * kNumEpiWarps : kNumEpiWarps;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes + kCombBytes;
  static_assert(kSubH % 1024 == 0, "H sub-block must keep 1024-byte atom alignment");
  static_assert((2 * kStages + 2 * kAccBufs + 1) * 8 + 16 <= kBarBytes, "barrier area too small");
  static_assert(kTmemCols <= 512, "tensor memory holds 512 columns");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// ---------------------------------------------------------------------------
// Epilogue helpers
// ---------------------------------------------------------------------------

// Four lanes with the same token >> 2 each hold the four Philox words of one
// column (lane i: column c + i, words for tokens 4q..4q+3).  Afterwards lane
// i holds, in w[m], the word of token 4q + i for column c + m.
__device__ __forceinline__ void quad_transpose(uint32_t (&w)[4], int lane) {
  const bool b0 = (lane & 1) != 0;
  const bool b1 = (lane & 2) != 0;
  const uint32_t s01 = b0 ? w[0] : w[1];
  const uint32_t s23 = b0 ? w[2] : w[3];
  const uint32_t r01 = __shfl_xor_sync(0xffffffffu, s01, 1);
  const uint32_t r23 = __shfl_xor_sync(0xffffffffu, s23, 1);
  if (b0) {
    w[0] = r01;
    w[2] = r23;
  } else {
    w[1] = r01;
    w[3] = r23;
  }
  const uint32_t s02 = b1 ? w[0] : w[2];
  const uint32_t s13 = b1 ? w[1] : w[3];
  const uint32_t r02 = __shfl_xor_sync(0xffffffffu, s02, 2);
  const uint32_t r13 = __shfl_xor_sync(0xffffffffu, s13, 2);
  if (b1) {
    w[0] = r02;
    w[1] = r13;
  } else {
    w[2] = r02;
    w[3] = r13;
  }
}

// Lane that ends up holding column j of a CW-column transpose-reduce.
template <int CW>
__device__ __forceinline__ int column_of_lane(int lane) {
  return CW == 32 ? lane : (lane >> 1);
}
template <int CW>
__device__ __forceinline__ int lane_of_column(int j) {
  return CW == 32 ? j : 2 * j;
}

// Transpose-reduce: every lane holds CW values (one per column); afterwards
// lane l holds the reduction over all 32 lanes of column column_of_lane(l).
// Each halving round keeps one half of the columns and trades the other half
// with the partner lane, so CW=32 costs 31 exchanges instead of 32 x 5.
struct OpMaxU64 {
  __device__ __forceinline__ static uint64_t apply(uint64_t a, uint64_t b) { return a > b ? a : b; }
};
struct OpMaxF {
  __device__ __forceinline__ static float apply(float a, float b) { return fmaxf(a, b); }
};
struct OpAddF {
  __device__ __forceinline__ static float apply(float a, float b) { return a + b; }
};

template <int CW, class Op, class T>
__device__ __forceinline__ T transpose_reduce(T (&k)[CW], int lane) {
#pragma unroll
  for (int half = CW / 2, off = 16; half >= 1; half /= 2, off /= 2) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const T send = upper ? k[i] : k[i + half];
      const T keep = upper ? k[i + half] : k[i];
      const T recv = __shfl_xor_sync(0xffffffffu, send, off);
      k[i] = Op::apply(keep, recv);
    }
  }
  if (CW == 16) k[0] = Op::apply(k[0], __shfl_xor_sync(0xffffffffu, k[0], 1));
  return k[0];
}

// 2^x with the hardware's approximate base-2 exponential (2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// lse_merge in base 2: sum 2^(x2 - m) = s, for x2 = x log2(e).
__device__ __forceinline__ void lse2_merge(float &m, float &s, float m2, float s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float mx = fmaxf(m, m2);
  s = s * ex2_approx(m - mx) + s2 * ex2_approx(m2 - mx);
  m = mx;
}

// Reads a published key from global memory, bypassing L1 (other CTAs update it).
__device__ __forceinline__ uint64_t ld_key(const unsigned long long *ptr) {
  return __ldcg(ptr);
}

// Noise words of one chunk: afterwards words[j] is the word of (row col0 + j,
// token v) for this lane's tile row v.  One Philox call per lane serves four
// consecutive tokens of one row; the quad transpose hands each lane its word.
template <int CW>
__device__ __forceinline__ void chunk_noise(const FmmsParams &p, int v, int col0, int lane,
                                            uint32_t tag, uint32_t (&words)[CW]) {
#pragma unroll
  for (int q4 = 0; q4 < CW / 4; ++q4) {
    const int colp = col0 + 4 * q4 + (lane & 3);  // column of this lane's Philox call
    const uint32_t bg = static_cast<uint32_t>(p.b_off + colp);
    uint64_t k64 = p.seed;
    if (p.row_seeds != nullptr && colp < p.B && FS_IN_BOUNDS(p.err, bg, p.rows_total))
      k64 = __ldg(p.row_seeds + bg);
    const Philox4 ph = philox4x32_10(static_cast<uint32_t>(v) >> 2, bg, p.step, tag,
                                     static_cast<uint32_t>(k64), static_cast<uint32_t>(k64 >> 32));
    uint32_t w[4] = {ph.w0, ph.w1, ph.w2, ph.w3};
    quad_transpose(w, lane);
#pragma unroll
    for (int m = 0; m < 4; ++m) words[4 * q4 + m] = w[m];
  }
}

// Transpose of the 32 x 32 bit matrix whose row r is lane r's x: afterwards
// lane c holds the bits c of every lane's x, lane r's bit at position r.
// Five rounds of swapping the off-diagonal blocks of size 16, 8, 4, 2, 1.
__device__ __forceinline__ uint32_t bit_transpose32(uint32_t x, int lane) {
  const uint32_t kMasks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int i = 0, sft = 16; i < 5; ++i, sft >>= 1) {
    const uint32_t m = kMasks[i];
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, sft);
    x = (lane & sft) ? ((x & ~m) | ((y >> sft) & m)) : ((x & m) | ((y & m) << sft));
  }
  return x;
}

// Bit j set when (row col0 + j, token v) is in range and, with a mask,
// allowed for that row.  Warp-collective: the warp's lanes hold 32
// consecutive tokens.  Lane j < CW gathers row col0 + j's 32 mask bits of
// those tokens (two words at most); a bit-matrix transpose then hands every
// lane its own token's bit of each row.
template <int CW>
__device__ __forceinline__ uint32_t chunk_allowed(const FmmsParams &p, int v, bool v_ok,
                                                  int col0, int lane) {
  const int n = p.B - col0;
  const uint32_t in_range = n >= CW ? ((1u << CW) - 1u) : ((1u << n) - 1u);
  if (p.mask == nullptr) return v_ok ? in_range : 0u;
  const int v0 = v - lane;  // token of lane 0 (a multiple of 8)
  uint32_t rowbits = 0u;
  if (lane < CW && lane < n && FS_IN_BOUNDS(p.err, p.b_off + col0 + lane, p.rows_total)) {
    const uint32_t *row = p.mask + static_cast<size_t>(p.b_off + col0 + lane) * p.mask_words;
    const int w0 = v0 >> 5;
    const int sh = v0 & 31;
    const uint32_t lo = w0 < p.mask_words ? __ldg(row + w0) : 0u;
    const uint32_t hi = (sh != 0 && w0 + 1 < p.mask_words) ? __ldg(row + w0 + 1) : 0u;
    rowbits = sh == 0 ? lo : ((lo >> sh) | (hi << (32 - sh)));
  }
  const uint32_t bits = bit_transpose32(rowbits, lane);
  return v_ok ? (bits & in_range) : 0u;
}

// Bit j set when (row col0 + j, token v) is in range, mask not consulted.
template <int CW>
__device__ __forceinline__ uint32_t chunk_in_range(const FmmsParams &p, bool v_ok, int col0) {
  if (!v_ok) return 0u;
  const int n = p.B - col0;
  return n >= CW ? ((1u << CW) - 1u) : ((1u << n) - 1u);
}

// Exact scores s = x + g of the allowed elements as packed keys,
// transpose-reduced into the lane's running best of its column.
template <int CW>
__device__ __forceinline__ void chunk_keys(const uint32_t (&acc)[CW], const uint32_t (&words)[CW],
                                           const FmmsParams &p, int v, uint32_t allowed, int lane,
                                           uint64_t &best) {
  uint64_t key[CW];
  const uint64_t low = 0xFFFFFFFFu - static_cast<uint32_t>(v);  // token part of the key
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const float s = fmaf(__uint_as_float(acc[j]), p.inv_temp, gumbel_from_u32(words[j]));
    const uint32_t hi = ((allowed >> j) & 1u) ? order_bits(__float_as_uint(s)) : 0u;
    key[j] = (static_cast<uint64_t>(hi) << 32) | low;
  }
  const uint64_t cmax = transpose_reduce<CW, OpMaxU64>(key, lane);
  best = cmax > best ? cmax : best;
}

// Log-sum-exp pieces, in base 2, of the allowed x2 = acc / T * log2(e) of one
// chunk (c1 = log2(e) / T), folded into the lane's running (m_run, s_run) of
// its column.  `ref` holds the running maxima of the chunk's CW columns
// (shared memory).  When every allowed element lies at most 60 above its
// column's running maximum, the chunk's terms are summed against those maxima
// as they stand: no maximum reduction, no broadcast, no rescaling (the sums
// stay below 2^75).  Otherwise (a segment's first chunk among them) the
// chunk's column maxima are reduced and merged.
template <int CW>
__device__ __forceinline__ void chunk_lse2(const uint32_t (&acc)[CW], float c1, uint32_t allowed,
                                           const float *ref, int lane, float &m_run,
                                           float &s_run) {
  float r[CW];
#pragma unroll
  for (int j4 = 0; j4 < CW / 4; ++j4) {
    const float4 v = reinterpret_cast<const float4 *>(ref)[j4];
    r[4 * j4 + 0] = v.x;
    r[4 * j4 + 1] = v.y;
    r[4 * j4 + 2] = v.z;
    r[4 * j4 + 3] = v.w;
  }
  float e[CW];
  bool over = false;
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const bool a = (allowed >> j) & 1u;
    const float dlt = fmaf(__uint_as_float(acc[j]), c1, -r[j]);
    over = over || (a && !(dlt <= 60.f));  // also a column with no maximum yet (+inf)
    e[j] = a ? ex2_approx(dlt) : 0.f;
  }
  if (!__any_sync(0xffffffffu, over)) {
    s_run += transpose_reduce<CW, OpAddF>(e, lane);
    return;
  }
  float xs[CW], t[CW];
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    xs[j] = ((allowed >> j) & 1u) ? __uint_as_float(acc[j]) * c1 : -INFINITY;
    t[j] = xs[j];
  }
  const float colmax = transpose_reduce<CW, OpMaxF>(t, lane);
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const float cm = __shfl_sync(0xffffffffu, colmax, lane_of_column<CW>(j));
    e[j] = (xs[j] == -INFINITY) ? 0.f : ex2_approx(xs[j] - cm);
  }
  const float colsum = transpose_reduce<CW, OpAddF>(e, lane);
  lse2_merge(m_run, s_run, colmax, colsum);
}

// The filter: may any element of the chunk (bit set in `cand`) reach its
// column's threshold?  The threshold of a column is the score of an element
// already computed exactly (the lane's own best, or the best any CTA has
// published for this row), so an element whose upper bound
// x + gumbel_upper_bound(r) is below it can be neither the maximum nor tied
// with it: skipping its exact score leaves the sampled token unchanged.
template <int CW>
__device__ __forceinline__ bool chunk_any_candidate(const uint32_t (&acc)[CW],
                                                    const uint32_t (&words)[CW],
                                                    const FmmsParams &p, uint32_t cand,
                                                    uint64_t best, uint64_t published, int lane) {
  const uint64_t k = published > best ? published : best;
  const float t_col = key_valid(k) ? __uint_as_float(key_score_bits(k)) : -INFINITY;
  bool any = false;
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const float thr = __shfl_sync(0xffffffffu, t_col, lane_of_column<CW>(j));
    const float ub = fmaf(__uint_as_float(acc[j]), p.inv_temp, gumbel_upper_bound(words[j]));
    any = any || (((cand >> j) & 1u) && ub >= thr);
  }
  return __any_sync(0xffffffffu, any);
}

// Fused vocabulary-parallel exchange, run by the epilogue threads of the
// last CTA of a rank's kernel (see TpArea): raise every rank's area to this
// rank's per-row maxima, count this rank in every area, and decode each area
// whose count this arrival completed.  `dec` is a shared-memory word;
// `failed`: some CTA of this call gave up on a bounded wait.
__device__ __forceinline__ void tp_exchange(const FmmsParams &p, int etid, int *dec, bool failed) {
  const int world = p.tp_world;
  const uint32_t par = p.tp_seq & 1u;
  if (etid == 0) *dec = 0;
  for (int i = etid; i < world * p.B; i += kEpiThreads) {
    const int q = i / p.B;
    const int b = i - q * p.B;
    const unsigned long long kb = __ldcg(p.keys + b);
    if (key_valid(kb)) atomicMax(&p.tp_area[q]->keys[par][b], kb);
  }
  if (failed)
    for (int q = etid; q < world; q += kEpiThreads) atomicOr(&p.tp_area[q]->err[par], 1u);
  __threadfence_system();
  sm100::epi_sync(kEpiThreads);
  for (int b = etid; b < p.B; b += kEpiThreads) p.keys[b] = 0ull;  // for this rank's next call
  if (etid < world) {
    __threadfence_system();
    const unsigned old = atomicAdd(&p.tp_area[etid]->arrivals[par], 1u);
    if (old == static_cast<unsigned>(world - 1)) atomicOr(dec, 1 << etid);
  }
  if (etid == 0) atomicExch(p.ticket, 0u);
  sm100::epi_sync(kEpiThreads);
  const int mine = *dec;
  for (int q = 0; q < world; ++q) {
    if (!((mine >> q) & 1)) continue;  // uniform across the CTA
    TpArea *a = p.tp_area[q];
    __threadfence_system();
    const bool bad = atomicAdd(&a->err[par], 0u) != 0u;
    for (int b = etid; b < p.B; b += kEpiThreads) {
      const unsigned long long kb = atomicExch(&a->keys[par][b], 0ull);
      a->tokens[par][b] = bad ? -1 : key_token(kb);
    }
    __threadfence_system();
    sm100::epi_sync(kEpiThreads);
    if (etid == 0) {
      atomicExch(&a->arrivals[par], 0u);
      if (bad) {
        atomicExch(&a->err[par], 0u);
        atomicExch(&a->failed, p.tp_seq + 1u);
      }
      __threadfence_system();
      sm100::st_release_sys(&a->flag, p.tp_seq + 1u);
    }
  }
}

// ---------------------------------------------------------------------------
// Roles
// ---------------------------------------------------------------------------

// Bytes of W a CTA loads per 64-wide K sub-block for `rows` rows from the
// tile start: 16 KB for a whole tile (one 128-row box, also for a tile cut
// short by fewer than 8 rows), else one kilobyte per 8-row granule (boxes of
// 64, 32, 16 and 8 rows).
__device__ __forceinline__ uint32_t w_sub_bytes(int rows) {
  if (rows <= 0) return 0u;
  if (rows >= kTileM) return static_cast<uint32_t>(kTileM * kBlockK * 2);
  return static_cast<uint32_t>((rows + kGranule - 1) / kGranule) * 1024u;
}

// Transposed pair tiles.  On a CTA pair with a 256-row batch tile, a tile of
// at most 240 vocabulary rows (a segment's partial tile) runs as logits^T:
// A = the pair's 256 batch rows of H (each CTA's 128, already staged), B =
// the tile's rows of W rounded up to n = a multiple of 16, n / 2 from each
// CTA, so the MMA costs n / 256 of a whole tile's instead of all of it.
// Accumulator lane = batch row, column j = vocabulary row tile.start + j.
// Returns n, or 0 for a tile that runs as usual.
template <int BN, bool PAIR>
__device__ __forceinline__ int transposed_cols(const Tile &t) {
  if constexpr (!PAIR || BN != 2 * kTileM) {
    return 0;
  } else {
    const int n = (t.hi - t.start + 15) & ~15;
    return n < BN ? n : 0;
  }
}

// The H loads of one stage (this CTA's rows of the batch operand).
template <int BN, int MODE, bool PAIR, bool MERGE = false>
__device__ __forceinline__ void issue_h(const CUtensorMap *th, const FmmsParams &p,
                                        uint8_t *stages, uint64_t *full, int stage, int sub0,
                                        int nsub, int rank, uint64_t pol_h) {
  using C = KCfg<BN, MODE, PAIR, MERGE>;
  uint8_t *sh0 = stages + stage * C::kStageBytes + C::kOffH;
  const uint32_t bar = PAIR ? sm100::cluster_addr(&full[stage], 0) : 0u;
#pragma unroll
  for (int j = 0; j < C::kSub; ++j) {
    if (j >= nsub) break;
    uint8_t *sh = sh0 + j * C::kSubH;
    const int x = (sub0 + j) * kBlockK;
    if constexpr (PAIR) {
      sm100::tma_load_2d_pair(sh, th, bar, x, p.b_off + rank * C::kHRows, pol_h);
    } else {
      sm100::tma_load_2d(sh, th, &full[stage], x, p.b_off, pol_h);
    }
  }
}

// TMA producer (one thread).  In pair mode both CTAs load their own half of
// every stage (128 W rows, BN/2 H rows) and count the bytes on the even
// CTA's full barrier; a freed stage is signalled to both CTAs by the even
// CTA's MMA commit (multicast to the pair).
template <int BN, int MODE, bool PAIR, bool MERGE = false>
__device__ __forceinline__ void role_producer(const CUtensorMap *tw, const PartMaps *twp,
                                              const CUtensorMap *th, const FmmsParams &p,
                                              const Schedule &sch, uint8_t *stages,
                                              uint64_t *full, uint64_t *empty,
                                              volatile int *abort_flag, int unit, int rank) {
  using C = KCfg<BN, MODE, PAIR, MERGE>;
  const uint64_t pol_w = sm100::l2_policy_evict_first();
  const uint64_t pol_h = sm100::l2_policy_evict_last();
  TileIter it(sch, unit, C::kMerge ? 1 : 0);
  Tile tile;
  int stage = 0;
  uint32_t phase = 0;
  long long issued = 0;
  // The H loads are gated in two cases: with a programmatic launch (p.pdl)
  // until the grid ahead in the stream has completed (H may be its output),
  // and in fs_sample_host (p.h_ready) until the copy of H from the host has
  // landed.  While the gate is closed, a stage's W loads go out at once and
  // its H loads are deferred as long as free stages remain, so the ring fills
  // with W meanwhile instead of stopping at the first stage.
  bool dep_pending = p.pdl != 0;
  int h_chunks_ready =  // chunks of H known to be loadable
      (p.h_ready != nullptr || dep_pending) ? -1 : 0x7FFFFFFF;
  int pend_stage[C::kStages], pend_sub0[C::kStages], pend_nsub[C::kStages];
  int npend = 0, pend_need = 0;
  // Opens the gate up to H chunk `need`: false if the copy of H did not land
  // within the wait limit.
  auto open_gate = [&](int need) -> bool {
    if (dep_pending) {
      sm100::grid_dependency_wait();
      dep_pending = false;
    }
    if (p.h_ready == nullptr) {
      h_chunks_ready = 0x7FFFFFFF;
      return true;
    }
    h_chunks_ready = need;
    return sm100::wait_flag_bounded(p.h_ready + need, p.h_epoch, abort_flag, p.err);
  };
  bool ok = p.test_no_loads == 0;
  while (ok && it.next(tile)) {
    const bool merged = C::kMerge && tile.pstart >= 0;
    const int tn = transposed_cols<BN, PAIR>(tile);
    Tile mine = PAIR ? pair_half(tile, rank) : tile;
    if (tn != 0) {  // each CTA of the pair: n / 2 rows from tile.start + rank n / 2
      mine.start = tile.start + rank * (tn / 2);
      mine.hi = mine.start + tn / 2;
    }
    const int rows = mine.hi - mine.start;
    const int nbox8 = rows > 0 ? (rows + kGranule - 1) / kGranule : 0;
    // 16 granules (a tile cut short by fewer than 8 rows at the end of a
    // segment) load as one 128-row box: the rows past the tile's end are in
    // bounds (the next segment's) or zero-filled past V, and masked anyway.
    const bool whole = nbox8 >= kTileM / kGranule;
    // A small partial tile (at most 32 rows) costs a whole tile's MMA loop
    // while streaming few W bytes: meanwhile the single-CTA kernel (the
    // bandwidth-bound batch sizes) prefetches the segment's next tile into
    // L2, so that its loads catch up.  (Larger partial tiles stream enough
    // themselves, and prefetching for them overflowed L2 on heads where every
    // CTA starts with one; on CTA pairs, tensor-bound, it only added traffic.)
    const int next_start = it.t < it.seg_hi ? it.t : -1;
    const bool prefetch_next = !PAIR && nbox8 <= 4 && next_start >= 0 && next_start < p.V;
    uint32_t sub_bytes = w_sub_bytes(rows) + C::kSubH + (merged ? C::kSubP : 0u);  // this CTA's
    if (PAIR) {
      const Tile other = pair_half(tile, 1 - rank);
      sub_bytes += (tn != 0 ? w_sub_bytes(tn / 2) : w_sub_bytes(other.hi - other.start)) + C::kSubH;
    }
    const int nks = (p.nk + C::kSub - 1) / C::kSub;
    for (int ks = 0; ks < nks; ++ks) {
      const int sub0 = ks * C::kSub;
      const int nsub = imin(C::kSub, p.nk - sub0);
      const uint32_t bytes = sub_bytes * static_cast<uint32_t>(nsub);
      if (!sm100::wait_bounded<PAIR>(&empty[stage], phase ^ 1u, abort_flag, p.err)) {
        ok = false;
        break;
      }
      uint8_t *sp0 = stages + stage * C::kStageBytes;
      uint8_t *sw0 = sp0 + C::kOffW;
      if (!PAIR || rank == 0) sm100::mbar_arrive_expect_tx(&full[stage], bytes);
      const uint32_t bar = PAIR ? sm100::cluster_addr(&full[stage], 0) : 0u;
      // W first: it never waits for H.
#pragma unroll
      for (int j = 0; j < C::kSub; ++j) {
        if (j >= nsub) break;
        uint8_t *sw = sw0 + j * C::kSubW;
        const int x = (sub0 + j) * kBlockK;
        if constexpr (C::kMerge) {
          // the merged partial's 8 rows, into this sub-block's P slot
          if (merged)
            sm100::tma_load_2d(sp0 + j * C::kSubP, &twp->box[0], &full[stage], x, tile.pstart,
                               pol_w);
        }
        if (whole) {
          if constexpr (PAIR) {
            sm100::tma_load_2d_pair(sw, tw, bar, x, mine.start, pol_w);
          } else {
            sm100::tma_load_2d(sw, tw, &full[stage], x, mine.start, pol_w);
          }
        } else {
          if (prefetch_next) sm100::tma_prefetch_2d(tw, x, next_start);
          // Boxes of 64, 32, 16 and 8 rows: the binary digits of the tile's
          // 8-row count, each at its 1024-byte-aligned place in the stage.
          int row = 0;
#pragma unroll
          for (int b = 3; b >= 0; --b) {
            if (!((nbox8 >> b) & 1)) continue;
            if constexpr (PAIR) {
              sm100::tma_load_2d_pair(sw + row * 128, &twp->box[b], bar, x, mine.start + row,
                                      pol_w);
            } else {
              sm100::tma_load_2d(sw + row * 128, &twp->box[b], &full[stage], x, mine.start + row,
                                 pol_w);
            }
            row += kGranule << b;
          }
        }
      }
      // Gate closed for the chunk of H this stage ends in: defer the stage's
      // H loads while free stages remain; then open it (wait) and issue every
      // deferred H load.  (The grid dependency cannot be polled, so with
      // p.pdl the gate opens once the ring is full or the CTA's stages end.)
      bool h_now = true;
      const int need = p.h_ready != nullptr ? (sub0 + nsub - 1) / p.h_chunk_subs : 0;
      if (need > h_chunks_ready) {
        pend_stage[npend] = stage;
        pend_sub0[npend] = sub0;
        pend_nsub[npend] = nsub;
        pend_need = need;
        ++npend;
        h_now = false;
        if (npend == C::kStages ||
            (!dep_pending && sm100::flag_is(p.h_ready + need, p.h_epoch))) {
          const bool landed = open_gate(need);
          // After a timeout too: the loads stay in bounds, and completing
          // the stages lets the drain below account for every copy.
          for (int q = 0; q < npend; ++q)
            issue_h<BN, MODE, PAIR, MERGE>(th, p, stages, full, pend_stage[q], pend_sub0[q],
                                           pend_nsub[q], rank, pol_h);
          npend = 0;
          if (!landed) {
            ok = false;
            ++issued;
            break;
          }
        }
      }
      if (h_now) issue_h<BN, MODE, PAIR, MERGE>(th, p, stages, full, stage, sub0, nsub, rank, pol_h);
      ++issued;
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  if (ok && npend > 0) {
    // The CTA's last stages are still waiting for H (a range shorter than the ring).
    const bool landed = open_gate(pend_need);
    for (int q = 0; q < npend; ++q)
      issue_h<BN, MODE, PAIR, MERGE>(th, p, stages, full, pend_stage[q], pend_sub0[q], pend_nsub[q], rank,
                              pol_h);
    npend = 0;
    ok = landed;
  }
  if (!ok && issued > 0 && (!PAIR || rank == 0)) {
    // Gave up: let the copies already in flight land before the CTA exits.
    // (The odd CTA of a pair cannot observe its copies, which complete on the
    // even CTA's barriers; it exits only after the cluster barrier at the end
    // of the kernel, which the even CTA reaches after this drain.)
    // One time limit covers the whole drain.
    const long long first = issued > C::kStages ? issued - C::kStages : 0;
    const long long t0 = clock64();
    for (long long n = first; n < issued; ++n) {
      const int s = static_cast<int>(n % C::kStages);
      const uint32_t ph = static_cast<uint32_t>((n / C::kStages) & 1);
      while (!sm100::mbar_try_wait<PAIR>(&full[s], ph) && clock64() - t0 < sm100::kWaitLimitCycles) {
      }
    }
  }
}

// MMA issuer (one thread; in pair mode only the even CTA's).
template <int BN, int MODE, bool PAIR, bool MERGE = false>
__device__ __forceinline__ void role_mma(const FmmsParams &p, const Schedule &sch,
                                         uint8_t *stages, uint64_t *full, uint64_t *empty,
                                         uint64_t *acc_full, uint64_t *acc_empty,
                                         uint64_t *drain_bar, uint32_t tmem_base,
                                         volatile int *abort_flag, int unit) {
  using C = KCfg<BN, MODE, PAIR, MERGE>;
  TileIter it(sch, unit, C::kMerge ? 1 : 0);
  Tile tile;
  int stage = 0;
  uint32_t phase = 0;
  int buf = 0;
  uint32_t acc_phase = 0;
  bool ok = true;
  const uint32_t stage_lo = sm100::desc_lo(sm100::smem_addr(stages));
  const uint32_t desc_hi = sm100::kDescHi;
  while (ok && it.next(tile)) {
    // A merged partial takes the next accumulator too.
    const bool merged = C::kMerge && tile.pstart >= 0;
    const int buf2 = buf + 1 == C::kAccBufs ? 0 : buf + 1;
    const uint32_t phase2 = buf + 1 == C::kAccBufs ? acc_phase ^ 1u : acc_phase;
    if (!sm100::wait_bounded<PAIR>(&acc_empty[buf], acc_phase ^ 1u, abort_flag, p.err)) break;
    if (merged && !sm100::wait_bounded<PAIR>(&acc_empty[buf2], phase2 ^ 1u, abort_flag, p.err))
      break;
    sm100::tc_fence_after();
    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
    const uint32_t d_tmem2 = tmem_base + static_cast<uint32_t>(buf2 * BN);
    // A transposed tile swaps the operands (H sub-blocks and W sub-blocks have
    // the same size there) and multiplies 256 x n.
    const int tn = transposed_cols<BN, PAIR>(tile);
    static_assert(!PAIR || BN != 2 * kTileM || C::kSubH == C::kSubW, "transposed operand strides");
    const uint32_t idesc = tn != 0 ? sm100::idesc_bf16_f32(2 * kTileM, tn) : C::kIdesc;
    const int nks = (p.nk + C::kSub - 1) / C::kSub;
    for (int ks = 0; ks < nks; ++ks) {
      if (!sm100::wait_bounded<PAIR>(&full[stage], phase, abort_flag, p.err)) {
        ok = false;
        break;
      }
      sm100::tc_fence_after();
      const int nsub = imin(C::kSub, p.nk - ks * C::kSub);
      // Descriptor low words of this stage's operands; each MMA below adds a
      // compile-time offset (in 16-byte units) to them.
      const uint32_t p_lo = stage_lo + static_cast<uint32_t>(stage * (C::kStageBytes >> 4));
      const uint32_t w_lo = p_lo + (C::kOffW >> 4);
      const uint32_t h_lo = p_lo + (C::kOffH >> 4);
      const uint32_t a_lo = tn != 0 ? h_lo : w_lo;
      const uint32_t b_lo = tn != 0 ? w_lo : h_lo;
      if (nsub == C::kSub) {
        // A full stage: every K step unrolled, only the tile's first MMA
        // overwrites the accumulator.
#pragma unroll
        for (int j = 0; j < C::kSub; ++j) {
#pragma unroll
          for (int kk = 0; kk < kBlockK / 16; ++kk) {
            const uint32_t acc = (j | kk) != 0 ? 1u : (ks != 0 ? 1u : 0u);
            sm100::mma_bf16_lo<PAIR>(d_tmem, a_lo + ((j * C::kSubW + kk * 32) >> 4),
                                     b_lo + ((j * C::kSubH + kk * 32) >> 4), desc_hi, idesc, acc);
          }
        }
      } else {
        // The tile's last stage, partly filled when d is not a multiple of
        // the stage's K extent.
#pragma unroll
        for (int j = 0; j < C::kSub; ++j) {
          if (j >= nsub) break;
#pragma unroll
          for (int kk = 0; kk < kBlockK / 16; ++kk) {
            const uint32_t acc = (ks | j | kk) != 0 ? 1u : 0u;
            sm100::mma_bf16_lo<PAIR>(d_tmem, a_lo + ((j * C::kSubW + kk * 32) >> 4),
                                     b_lo + ((j * C::kSubH + kk * 32) >> 4), desc_hi, idesc, acc);
          }
        }
      }
      if constexpr (C::kMerge) {
        // The merged partial: rows 0-7 from its P slot; rows 8-127 of the
        // operand run on into the rest of the stage and land in accumulator
        // rows the epilogue never reads.
        if (merged) {
#pragma unroll
          for (int j = 0; j < C::kSub; ++j) {
            if (j >= nsub) break;
#pragma unroll
            for (int kk = 0; kk < kBlockK / 16; ++kk) {
              sm100::mma_bf16_lo<false>(d_tmem2, p_lo + ((j * C::kSubP + kk * 32) >> 4),
                                        b_lo + ((j * C::kSubH + kk * 32) >> 4), desc_hi,
                                        C::kIdesc, (ks | j | kk) != 0 ? 1u : 0u);
            }
          }
        }
      }
      // Frees the stage (in both CTAs of a pair) once these MMAs finish.
      if constexpr (PAIR) {
        sm100::mma_commit_pair_both(&empty[stage]);
      } else {
        sm100::mma_commit(&empty[stage]);
      }
      if (++stage == C::kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    // Accumulator ready for the epilogue (of both CTAs of a pair).
    if constexpr (PAIR) {
      sm100::mma_commit_pair_both(&acc_full[buf]);
    } else {
      sm100::mma_commit(&acc_full[buf]);
      if (merged) sm100::mma_commit(&acc_full[buf2]);
    }
    for (int n = merged ? 2 : 1; n > 0; --n) {
      if (++buf == C::kAccBufs) {
        buf = 0;
        acc_phase ^= 1u;
      }
    }
  }
  // Drain: every MMA issued above has completed once this arrives.
  if constexpr (PAIR) {
    sm100::mma_commit_pair(drain_bar);
  } else {
    sm100::mma_commit(drain_bar);
  }
  const long long t0 = clock64();
  while (!sm100::mbar_try_wait<PAIR>(drain_bar, 0) && clock64() - t0 < sm100::kWaitLimitCycles) {
  }
}

// Mask bits of row b (of this launch) for the 4 tokens from vg0 (a multiple
// of 4, so they lie in one mask word): bit m for token vg0 + m; all set
// without a mask.
__device__ __forceinline__ uint32_t row_mask4(const FmmsParams &p, int b, int vg0) {
  if (p.mask == nullptr) return 0xFu;
  const int w = vg0 >> 5;
  if (!FS_IN_BOUNDS(p.err, p.b_off + b, p.rows_total) || w >= p.mask_words) return 0u;
  return (__ldg(p.mask + static_cast<size_t>(p.b_off + b) * p.mask_words + w) >> (vg0 & 31)) & 0xFu;
}

// The Philox key of row b: its own seed, or the call's.
__device__ __forceinline__ uint64_t row_key64(const FmmsParams &p, int b) {
  const uint32_t bg = static_cast<uint32_t>(p.b_off + b);
  if (p.row_seeds != nullptr && FS_IN_BOUNDS(p.err, bg, p.rows_total)) return __ldg(p.row_seeds + bg);
  return p.seed;
}

// Best packed key of row b over the 4 tokens from vg0 (a multiple of 4) whose
// bit is set in `allowed`, with noise tag `tag`: one Philox call, whose word
// m is token vg0 + m's (the words chunk_noise hands out).  The filter of
// chunk_any_candidate comes first: only when some element's upper bound
// reaches the score of `thr_key` (computed exactly) are the exact scores
// computed.  0 when none passes.
__device__ __forceinline__ uint64_t row_best4(const uint32_t (&acc)[4], const FmmsParams &p, int b,
                                              int vg0, uint32_t tag, uint64_t k64,
                                              uint32_t allowed, uint64_t thr_key) {
  const Philox4 ph = philox4x32_10(static_cast<uint32_t>(vg0) >> 2, static_cast<uint32_t>(p.b_off + b),
                                   p.step, tag, static_cast<uint32_t>(k64),
                                   static_cast<uint32_t>(k64 >> 32));
  const uint32_t w[4] = {ph.w0, ph.w1, ph.w2, ph.w3};
  const float thr = key_valid(thr_key) ? __uint_as_float(key_score_bits(thr_key)) : -INFINITY;
  bool any = false;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float ub = fmaf(__uint_as_float(acc[m]), p.inv_temp, gumbel_upper_bound(w[m]));
    any = any || (((allowed >> m) & 1u) && ub >= thr);
  }
  if (!any) return 0ull;
  uint64_t best = 0ull;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    if (!((allowed >> m) & 1u)) continue;
    const float sc = fmaf(__uint_as_float(acc[m]), p.inv_temp, gumbel_from_u32(w[m]));
    const uint64_t key = pack_key(__float_as_uint(sc), vg0 + m);
    best = key > best ? key : best;
  }
  return best;
}

// Mask bits of row b (of this launch) for the 16 tokens from vg0 (a multiple
// of 8): bit j for token vg0 + j; all set without a mask.
__device__ __forceinline__ uint32_t row_mask16(const FmmsParams &p, int b, int vg0) {
  if (p.mask == nullptr) return 0xFFFFu;
  if (!FS_IN_BOUNDS(p.err, p.b_off + b, p.rows_total)) return 0u;
  const uint32_t *row = p.mask + static_cast<size_t>(p.b_off + b) * p.mask_words;
  const int w0 = vg0 >> 5;
  const int sh = vg0 & 31;
  const uint32_t lo = w0 < p.mask_words ? __ldg(row + w0) : 0u;
  const uint32_t hi = (sh > 16 && w0 + 1 < p.mask_words) ? __ldg(row + w0 + 1) : 0u;
  return (sh == 0 ? lo : ((lo >> sh) | (hi << (32 - sh)))) & 0xFFFFu;
}

// Best packed key of row b over the 16 tokens from vg0 (a multiple of 8)
// whose bit is set in `allowed`, noise tag `tag`: the filter over all 16
// first (four Philox calls, word m of call i for token vg0 + 4 i + m), then,
// only when some upper bound reaches the score of `thr_key`, the exact scores
// of the groups of four that hold an allowed token, their noise drawn again.
// 0 when none passes.  The exact pass is a loop that is not unrolled: it
// runs rarely, and indexing acc in it keeps acc in local memory there instead
// of in registers that the hot path needs.
__device__ __forceinline__ uint64_t row_best16(const uint32_t (&acc)[16], const FmmsParams &p,
                                               int b, int vg0, uint32_t tag, uint64_t k64,
                                               uint32_t allowed, uint64_t thr_key) {
  const float thr = key_valid(thr_key) ? __uint_as_float(key_score_bits(thr_key)) : -INFINITY;
  bool any = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const Philox4 ph = philox4x32_10((static_cast<uint32_t>(vg0) >> 2) + static_cast<uint32_t>(i),
                                     static_cast<uint32_t>(p.b_off + b), p.step, tag,
                                     static_cast<uint32_t>(k64), static_cast<uint32_t>(k64 >> 32));
    const uint32_t w[4] = {ph.w0, ph.w1, ph.w2, ph.w3};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float ub = fmaf(__uint_as_float(acc[4 * i + m]), p.inv_temp, gumbel_upper_bound(w[m]));
      any = any || (((allowed >> (4 * i + m)) & 1u) && ub >= thr);
    }
  }
  if (!any) return 0ull;
  uint64_t best = 0ull;
#pragma unroll 1
  for (int i = 0; i < 4; ++i) {
    if (((allowed >> (4 * i)) & 0xFu) == 0u) continue;
    const Philox4 ph = philox4x32_10((static_cast<uint32_t>(vg0) >> 2) + static_cast<uint32_t>(i),
                                     static_cast<uint32_t>(p.b_off + b), p.step, tag,
                                     static_cast<uint32_t>(k64), static_cast<uint32_t>(k64 >> 32));
    const uint32_t w[4] = {ph.w0, ph.w1, ph.w2, ph.w3};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int j = 4 * i + m;
      if (!((allowed >> j) & 1u)) continue;
      const float sc = fmaf(__uint_as_float(acc[j]), p.inv_temp, gumbel_from_u32(w[m]));
      const uint64_t key = pack_key(__float_as_uint(sc), vg0 + j);
      best = key > best ? key : best;
    }
  }
  return best;
}

// Grouped-mode epilogue of a transposed pair tile (see transposed_cols): the
// thread owns batch row b (its TMEM lane) and walks the tile's n columns in
// 16-column chunks (h, h + 4, ... among the warps of its lane quarter), with
// no exchange between lanes, and folds the row's (best key, max, sum) over the
// tile into comb slot h of column b.  The tile is the first of its segment;
// the caller synchronises the epilogue warps before the next tile reads the
// slots.  (In this mode 16-column chunks ran faster than four-column ones.)
template <int BN>
__device__ __forceinline__ void epi_transposed_grouped(const FmmsParams &p, const Tile &t, int tn,
                                                       uint32_t tbase, int b, int h, int unit,
                                                       float c1, uint64_t *comb_key,
                                                       float *comb_m, float *comb_s) {
  constexpr int kWpq = kNumEpiWarps / 4;
  const bool row_ok = b < p.B;
  const uint64_t k64 = row_ok ? row_key64(p, b) : 0ull;
  uint64_t g_best = 0ull;
  float g_m = -INFINITY, g_s = 0.f;
  unsigned long long *gk = nullptr;
  const long long gki = static_cast<long long>(t.slot - unit) * p.B + b;
  if (p.gkeys != nullptr && row_ok && FS_IN_BOUNDS(p.err, gki, p.gkeys_cap)) gk = p.gkeys + gki;
  uint64_t g_pub = 0ull;
  for (int col0 = 16 * h; col0 < tn; col0 += 16 * kWpq) {  // warp-uniform
    uint32_t acc[16];
    if (!FS_IN_BOUNDS(p.err, col0 + 15, BN)) continue;
    sm100::tmem_ld_16(tbase + col0, acc);
    sm100::tmem_wait_ld();
    if (!row_ok) continue;
    const int v0 = t.start + col0;
    uint32_t in_range = 0u;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (v0 + j >= t.lo && v0 + j < t.hi) in_range |= 1u << j;
    if (in_range == 0u) continue;
    const int vg0 = v0 + p.vocab_offset;
    const uint32_t allowed = in_range & row_mask16(p, b, vg0);
    // log-sum-exp pieces in base 2
    float cm = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if ((allowed >> j) & 1u) cm = fmaxf(cm, __uint_as_float(acc[j]) * c1);
    if (cm != -INFINITY) {
      float cs = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if ((allowed >> j) & 1u) cs += ex2_approx(__uint_as_float(acc[j]) * c1 - cm);
      lse2_merge(g_m, g_s, cm, cs);
    }
    if (gk != nullptr && g_pub == 0ull) g_pub = ld_key(gk);
    const uint64_t best =
        row_best16(acc, p, b, vg0, 0u, k64, allowed, g_pub > g_best ? g_pub : g_best);
    if (key_valid(best) && best > g_best) g_best = best;
  }
  if (row_ok) {
    if (gk != nullptr && key_valid(g_best) && g_best > g_pub)
      atomicMax(gk, static_cast<unsigned long long>(g_best));
    const int si = h * BN + b;
    if (g_best > comb_key[si]) comb_key[si] = g_best;
    float m = comb_m[si], s = comb_s[si];
    lse2_merge(m, s, g_m, g_s);
    comb_m[si] = m;
    comb_s[si] = s;
  }
}

// Flat-mode epilogue of a transposed pair tile (see transposed_cols): the
// thread owns batch row b (its TMEM lane) and walks the tile's n columns four
// at a time, the warps of a lane quarter taking 16-column chunks in turn (h,
// h + 4, ...), with no exchange between lanes; each sample's row maximum is
// published at once.  Four columns at a time keep this cold path within a few
// registers: it shares the kernel's register budget with the hot one.
template <int BN>
__device__ __forceinline__ void epi_transposed_flat(const FmmsParams &p, const Tile &t, int tn,
                                                    uint32_t tbase, int b, int h) {
  constexpr int kWpq = kNumEpiWarps / 4;
  const bool row_ok = b < p.B;
  const uint64_t k64 = row_ok ? row_key64(p, b) : 0ull;
#pragma unroll 1
  for (int c = 16 * h; c < tn; c += (c & 15) == 12 ? 16 * kWpq - 12 : 4) {  // warp-uniform
    uint32_t acc[4];
    if (!FS_IN_BOUNDS(p.err, c + 3, BN)) continue;
    sm100::tmem_ld_4(tbase + c, acc);
    sm100::tmem_wait_ld();
    const int v0 = t.start + c;
    uint32_t allowed = 0u;
#pragma unroll
    for (int m = 0; m < 4; ++m)
      if (row_ok && v0 + m >= t.lo && v0 + m < t.hi) allowed |= 1u << m;
    if (allowed == 0u) continue;
    const int vg0 = v0 + p.vocab_offset;
    allowed &= row_mask4(p, b, vg0);
    if (allowed == 0u) continue;
#pragma unroll 1
    for (int smp = 0; smp < p.num_samples; ++smp) {
      if (!FS_IN_BOUNDS(p.err, smp * kMaxBN + b, p.keys_cap)) continue;
      unsigned long long *kp = p.keys + smp * kMaxBN + b;
      const uint64_t pub = ld_key(kp);
      const uint64_t best =
          row_best4(acc, p, b, vg0, 2u * static_cast<uint32_t>(smp), k64, allowed, pub);
      if (key_valid(best) && best > pub) atomicMax(kp, static_cast<unsigned long long>(best));
    }
  }
}

// Epilogue warps.  In pair mode each CTA drains its own 128 accumulator rows
// (its half of the pair tile); the even CTA's MMA commit signals a filled
// accumulator to both CTAs, and the odd CTA's warps release it on the even
// CTA's barrier, where the MMAs are issued.
template <int BN, int MODE, bool PAIR, bool MERGE = false>
__device__ __forceinline__ void role_epilogue(const FmmsParams &p, const Schedule &sch,
                                              uint32_t tmem_base, uint64_t *acc_full,
                                              uint64_t *acc_empty, volatile int *abort_flag,
                                              int *last_flag, uint64_t *comb_key, float *comb_m,
                                              float *comb_s, int warp, int lane, int unit,
                                              int rank) {
  using C = KCfg<BN, MODE, PAIR, MERGE>;
  constexpr int CW = C::kCW;
  const int q = warp & 3;          // TMEM lane quarter this warp may access
  const int h = (warp - 2) >> 2;   // which of the quarter's warps: chunks h, h+4, ...
  const float c1 = p.inv_temp * 1.4426950408889634f;  // log2(e) / T: base-2 log-sum-exp
  const int etid = (warp - 2) * 32 + lane;
  const bool has_chunks = h < C::kChunks;
  // A programmatic launch may start while the grid ahead in the stream (the
  // previous call, which shares the workspace) finishes: touch no global
  // memory before it has completed.  Returns at once otherwise.
  if (p.pdl) sm100::grid_dependency_wait();

  // Grouped mode: the running (best key, max, sum) of each (lane quarter,
  // column) over the current segment live in shared memory, [4][BN] each,
  // which keeps them out of the registers the chunk arithmetic needs.
  if constexpr (MODE == kModeGrouped) {
    for (int i = etid; i < 4 * BN; i += kEpiThreads) {
      comb_key[i] = 0ull;
      comb_m[i] = -INFINITY;
      comb_s[i] = 0.f;
    }
    sm100::epi_sync(kEpiThreads);
  }

  TileIter it(sch, unit, C::kMerge ? 1 : 0);
  Tile tile;
  int buf = 0;
  uint32_t phase = 0;
  bool aborted = false;
  // One accumulator: wait for it, run the chunk pipeline over it, hand it back.
  auto run_acc = [&](const Tile &cur) {
    // After an abort the loop keeps walking the tiles without touching TMEM,
    // so that every epilogue warp reaches the same named barriers.  The
    // decision is made warp-uniform because the TMEM loads below are
    // warp-collective.
    const bool got = aborted ? false : sm100::wait_bounded<PAIR>(&acc_full[buf], phase, abort_flag, p.err);
    aborted = __any_sync(0xffffffffu, !got);
    const int tn = transposed_cols<BN, PAIR>(cur);
    if (!aborted && tn != 0) {
      sm100::tc_fence_after();
      if constexpr (MODE != kModeLogits) {
        const uint32_t tb =
            tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * BN);
        const int b = rank * kTileM + 32 * q + lane;  // this thread's batch row
        if constexpr (MODE == kModeGrouped) {
          epi_transposed_grouped<BN>(p, cur, tn, tb, b, h, unit, c1, comb_key, comb_m, comb_s);
        } else {
          epi_transposed_flat<BN>(p, cur, tn, tb, b, h);
        }
      }
    } else if (!aborted) {
      sm100::tc_fence_after();
      const Tile mine = PAIR ? pair_half(cur, rank) : cur;
      const int v = mine.start + 32 * q + lane;           // row of W in this launch
      const bool v_ok = v >= mine.lo && v < mine.hi;
      const int vg = v + p.vocab_offset;                  // global token index
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * BN);
#pragma unroll
      for (int kk = 0; kk < C::kChunksPerWarp; ++kk) {
        if (!has_chunks) continue;
        const int k = kk * C::kWarpsPerQuarter + h;
        const int col0 = k * CW;
        if (col0 >= p.B) continue;  // warp-uniform
        uint32_t acc[CW];
        if (!FS_IN_BOUNDS(p.err, buf * BN + col0 + CW - 1, C::kTmemCols)) continue;  // warp-uniform
        if constexpr (CW == 32) {
          sm100::tmem_ld_32(tbase + col0, acc);
        } else {
          sm100::tmem_ld_16(tbase + col0, acc);
        }
        sm100::tmem_wait_ld();
        if constexpr (MODE == kModeLogits) {
          if (v_ok) {
            float *dst = p.logits + static_cast<size_t>(col0) * p.V + v;
            const int ncol = imin(CW, p.B - col0);
#pragma unroll
            for (int j = 0; j < CW; ++j) {
              if (j < ncol &&
                  FS_IN_BOUNDS(p.err, static_cast<long long>(col0 + j) * p.V + v, p.logits_cap))
                *dst = __uint_as_float(acc[j]);
              dst += p.V;
            }
          }
        } else {
          const int c = col0 + column_of_lane<CW>(lane);  // this lane's column
          if constexpr (MODE == kModeFlat) {
            // Sample smp draws with token-noise tag 2 smp and keeps its running
            // per-row maximum in the published keys [smp][row]: every exact
            // chunk raises it at once, which also sharpens every CTA's filter.
            // The mask is consulted only on the exact path.
            const uint32_t in_range = chunk_in_range<CW>(p, v_ok, col0);
            uint32_t allowed = 0u;
            bool have_allowed = false;
#pragma unroll 1
            for (int smp = 0; smp < p.num_samples; ++smp) {
              unsigned long long *kp = p.keys + smp * kMaxBN + c;
              const bool kin = c < p.B && FS_IN_BOUNDS(p.err, smp * kMaxBN + c, p.keys_cap);
              const uint64_t pub = kin ? ld_key(kp) : 0ull;  // in flight during Philox
              uint32_t words[CW];
              chunk_noise<CW>(p, vg, col0, lane, 2u * static_cast<uint32_t>(smp), words);
              if (chunk_any_candidate<CW>(acc, words, p, in_range, 0ull, pub, lane)) {
                if (!have_allowed) {
                  allowed = chunk_allowed<CW>(p, vg, v_ok, col0, lane);
                  have_allowed = true;
                }
                uint64_t cbest = 0ull;
                chunk_keys<CW>(acc, words, p, vg, allowed, lane, cbest);
                if ((lane & 1) == 0 && kin && key_valid(cbest) && cbest > pub)
                  atomicMax(kp, static_cast<unsigned long long>(cbest));
              }
            }
          } else {
            const long long gki = static_cast<long long>(tile.slot - unit) * p.B + c;
            unsigned long long *gk =
                (p.gkeys && (c >= p.B || FS_IN_BOUNDS(p.err, gki, p.gkeys_cap))) ? p.gkeys + gki
                                                                              : nullptr;
            const uint64_t pub = (gk != nullptr && c < p.B) ? ld_key(gk) : 0ull;
            const uint32_t allowed = chunk_allowed<CW>(p, vg, v_ok, col0, lane);
            uint32_t words[CW];
            chunk_noise<CW>(p, vg, col0, lane, 0u, words);
            // this lane's (quarter, column) state
            const int si = FS_IN_BOUNDS(p.err, q * BN + c, 4 * BN) ? q * BN + c : 0;
            float m_run = comb_m[si], s_run = comb_s[si];
            uint64_t best = comb_key[si];
            chunk_lse2<CW>(acc, c1, allowed, comb_m + q * BN + col0, lane, m_run, s_run);
            if (chunk_any_candidate<CW>(acc, words, p, allowed, best, pub, lane)) {
              chunk_keys<CW>(acc, words, p, vg, allowed, lane, best);
              if (gk != nullptr && (lane & 1) == 0 && c < p.B && key_valid(best) && best > pub)
                atomicMax(gk, static_cast<unsigned long long>(best));
            }
            if ((lane & 1) == 0) {  // the two lanes of a column hold the same values
              comb_key[si] = best;
              comb_m[si] = m_run;
              comb_s[si] = s_run;
            }
          }
        }
      }
    }
    if (!aborted) {
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && rank == 1) {
          sm100::mbar_arrive_cluster(sm100::cluster_addr(&acc_empty[buf], 0));
        } else {
          sm100::mbar_arrive(&acc_empty[buf]);
        }
      }
    }
    if (++buf == C::kAccBufs) {
      buf = 0;
      phase ^= 1u;
    }
  };
  while (it.next(tile)) {
    run_acc(tile);
    // A merged partial comes as a second accumulator after its whole tile.
    if (C::kMerge && tile.pstart >= 0) run_acc(partial_of(tile));
    // A transposed tile wrote other warps' slots of the segment's state.
    if (MODE == kModeGrouped && transposed_cols<BN, PAIR>(tile) != 0) sm100::epi_sync(kEpiThreads);

    if constexpr (MODE == kModeGrouped) {
      if (tile.last) {
        // Segment done: combine the four lane quarters, write the partial
        // (slot per CTA: a pair's two CTAs write slots 2 s and 2 s + 1) and
        // reset the state for the next segment.
        sm100::epi_sync(kEpiThreads);
        const size_t slot = PAIR ? 2 * static_cast<size_t>(tile.slot) + rank
                                 : static_cast<size_t>(tile.slot);
        for (int b = etid; b < BN; b += kEpiThreads) {
          uint64_t kb = 0ull;
          float m = -INFINITY, s = 0.f;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const uint64_t kq = comb_key[qq * BN + b];
            kb = kq > kb ? kq : kb;
            lse2_merge(m, s, comb_m[qq * BN + b], comb_s[qq * BN + b]);
            comb_key[qq * BN + b] = 0ull;
            comb_m[qq * BN + b] = -INFINITY;
            comb_s[qq * BN + b] = 0.f;
          }
          if (b < p.B && !*abort_flag &&
              FS_IN_BOUNDS(p.err, static_cast<long long>(slot) * p.B + b, p.partials_cap)) {
            GroupPartial gp;
            gp.key = kb;
            gp.m = m * 0.69314718055994531f;  // base-2 maximum back to natural units
            gp.sum = s;
            p.partials[slot * p.B + b] = gp;
          }
        }
        sm100::epi_sync(kEpiThreads);
      }
    }
  }

  if (MODE == kModeFlat && p.no_ticket) return;  // a second kernel decodes the keys
  if constexpr (MODE == kModeFlat) {
    // Every maximum is already published; take a ticket, and the last CTA
    // decodes the keys and re-zeroes them for the next call.  With the fused
    // exchange an aborted CTA counts itself too (in the ticket's high half),
    // so that the exchange still completes, marked as failed, and no peer's
    // wait for the tokens runs into its time limit.
    __threadfence();
    sm100::epi_sync(kEpiThreads);
    if (etid == 0) {
      int last = 0;
      if (p.tp_world > 0) {
        const unsigned inc = *abort_flag ? 0x10000u : 1u;
        const unsigned old = atomicAdd(p.ticket, inc);
        const unsigned failed = (old >> 16) + (inc >> 16);
        if ((old & 0xFFFFu) + (old >> 16) + 1u == static_cast<unsigned>(p.num_ctas))
          last = failed ? 2 : 1;
      } else if (!*abort_flag) {
        last = (atomicAdd(p.ticket, 1u) == static_cast<unsigned>(p.num_ctas - 1)) ? 1 : 0;
      }
      *last_flag = last;
    }
    sm100::epi_sync(kEpiThreads);
    if (*last_flag && p.tp_world > 0) {
      __threadfence();
      tp_exchange(p, etid, last_flag + 1, *last_flag == 2);
    } else if (*last_flag) {
      __threadfence();
      const int total = p.B * p.num_samples;
      for (int i = etid; i < total; i += kEpiThreads) {
        const int b = i / p.num_samples;
        const int smp = i - b * p.num_samples;
        if (!FS_IN_BOUNDS(p.err, smp * kMaxBN + b, p.keys_cap) ||
            !FS_IN_BOUNDS(p.err, i, p.out_cap))
          continue;
        const unsigned long long kb = atomicExch(p.keys + smp * kMaxBN + b, 0ull);
        if (p.out_keys != nullptr)
          p.out_keys[i] = static_cast<long long>(kb ^ 0x8000000000000000ull);  // signed order
        else
          p.out_idx[i] = key_token(kb);
      }
      if (etid == 0) atomicExch(p.ticket, 0u);
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------
template <int BN, int MODE, bool PAIR, bool MERGE = false>
__global__ void __launch_bounds__(kThreads, 1)
    fmms_kernel(const __grid_constant__ CUtensorMap tmap_w,
                const __grid_constant__ PartMaps tmap_wp,
                const __grid_constant__ CUtensorMap tmap_h, const FmmsParams p) {
  using C = KCfg<BN, MODE, PAIR, MERGE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kStages * C::kStageBytes);
  uint64_t *full = bars;
  uint64_t *empty = full + C::kStages;
  uint64_t *acc_full = empty + C::kStages;
  uint64_t *acc_empty = acc_full + C::kAccBufs;
  uint64_t *drain_bar = acc_empty + C::kAccBufs;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *last_flag = reinterpret_cast<int *>(tmem_slot + 2);  // tmem_slot + 3: exchange word
  uint8_t *comb = reinterpret_cast<uint8_t *>(bars) + C::kBarBytes;
  uint64_t *comb_key = reinterpret_cast<uint64_t *>(comb);
  float *comb_m = reinterpret_cast<float *>(comb_key + 4 * BN);
  float *comb_s = comb_m + 4 * BN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Pair mode: the two CTAs of a cluster form schedule unit blockIdx.x / 2.
  const int rank = PAIR ? static_cast<int>(sm100::cluster_ctarank()) : 0;
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  Schedule sch;
  sch.V = p.V;
  sch.G = p.G;
  sch.num_ctas = PAIR ? p.num_ctas / 2 : p.num_ctas;
  sch.ngran = p.ngran;
  sch.tile_rows = PAIR ? 2 * kTileM : kTileM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      sm100::mbar_init(&acc_full[b], 1);
      sm100::mbar_init(&acc_empty[b], C::kEpiArrivals);
    }
    sm100::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *last_flag = 0;
    sm100::fence_mbar_init();
    sm100::fence_async_smem();
    sm100::prefetch_tensormap(&tmap_w);
#pragma unroll
    for (int b = 0; b < 4; ++b) sm100::prefetch_tensormap(&tmap_wp.box[b]);
    sm100::prefetch_tensormap(&tmap_h);
  }
  if constexpr (PAIR) {
    // Both CTAs' barriers are initialised before either CTA signals the
    // other's; the pair then allocates tensor memory collectively.
    __syncthreads();
    sm100::cluster_sync();
    if (warp == 1) {
      sm100::tmem_alloc_pair(tmem_slot, C::kTmemCols);
      sm100::tmem_relinquish_pair();
    }
  } else {
    if (warp == 1) {
      sm100::tmem_alloc(tmem_slot, C::kTmemCols);
      sm100::tmem_relinquish();
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0)
      role_producer<BN, MODE, PAIR, MERGE>(&tmap_w, &tmap_wp, &tmap_h, p, sch, stages, full, empty,
                                    abort_flag, unit, rank);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0)
      role_mma<BN, MODE, PAIR, MERGE>(p, sch, stages, full, empty, acc_full, acc_empty, drain_bar,
                               tmem_base, abort_flag, unit);
    __syncwarp();
  } else {
    role_epilogue<BN, MODE, PAIR, MERGE>(p, sch, tmem_base, acc_full, acc_empty, abort_flag, last_flag,
                                  comb_key, comb_m, comb_s, warp, lane, unit, rank);
  }

  // The group merge or the logits sampler that follows may start launching.
  sm100::launch_dependents();
  sm100::tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // Neither CTA frees tensor memory while the other may still use it: the
    // even CTA's MMAs write both, and each CTA's epilogue reads its own.
    sm100::cluster_sync();
  }
  sm100::tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) {
      sm100::tmem_dealloc_pair(tmem_base, C::kTmemCols);
    } else {
      sm100::tmem_dealloc(tmem_base, C::kTmemCols);
    }
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
// p.pdl: launched with programmatic stream serialization, so the kernel may
// start while the kernel ahead of it in the stream finishes (that kernel's
// CTAs signal launch_dependents once their work is done); it streams W at
// once and waits for the grid dependency before it loads H or touches the
// workspace.
template <int BN, int MODE, bool MERGE = false>
cudaError_t launch_t(const CUtensorMap &tw, const PartMaps &twp, const CUtensorMap &th,
                            const FmmsParams &p, cudaStream_t stream) {
  using C = KCfg<BN, MODE, false, MERGE>;
  auto kern = fmms_kernel<BN, MODE, false, MERGE>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.num_ctas), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, tw, twp, th, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Pair kernels: clusters of two CTAs, p.num_ctas = 2 x schedule units.
template <int BN, int MODE>
cudaLaunchConfig_t pair_config(int num_ctas, cudaStream_t stream,
                                      cudaLaunchAttribute *attr, bool pdl = false) {
  using C = KCfg<BN, MODE, true>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_ctas), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cfg;
}

template <int BN, int MODE>
cudaError_t pair_units_t(int *units) {
  using C = KCfg<BN, MODE, true>;
  auto kern = fmms_kernel<BN, MODE, true>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config<BN, MODE>(2, nullptr, attr);
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
  if (e != cudaSuccess) return e;
  *units = n;
  return cudaSuccess;
}

template <int BN, int MODE>
cudaError_t launch_pair_t(const CUtensorMap &tw, const PartMaps &twp,
                                 const CUtensorMap &th, const FmmsParams &p,
                                 cudaStream_t stream) {
  using C = KCfg<BN, MODE, true>;
  auto kern = fmms_kernel<BN, MODE, true>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config<BN, MODE>(p.num_ctas, stream, attr, p.pdl != 0);
  e = cudaLaunchKernelEx(&cfg, kern, tw, twp, th, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fmms
