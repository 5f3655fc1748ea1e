// aux_kernels.cu -- the small kernels around the fused one:
//  * the Group-Gumbel-Max merge of per-(segment, row) partials (readus.org
//    page, "Group Gumbel Max": pick a group with Gumbel noise on the group
//    log-masses, then take the sample inside the winning group);
//  * the second kernel of the unfused mode, sampling from fp32 logits in HBM;
//  * test kernels exposing the device Philox and Gumbel primitives.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fmms.h"
#include "fmms_common.cuh"
#include "launch.h"
#include "noise.cuh"
#include "sm100.cuh"

namespace fmms {

// Launches `kern` with programmatic stream serialization: it may be scheduled
// while the kernel ahead of it is finishing, and waits for that kernel with
// grid_dependency_wait() before touching its results.
template <typename... KArgs, typename... Args>
static cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block,
                                    cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---------------------------------------------------------------------------
// Group merge: one warp per row; lanes stride over the groups.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) group_merge_kernel(const MergeParams m) {
  sm100::grid_dependency_wait();  // the fused kernel's partials
  const int b = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= m.B) return;
  Schedule sch;
  sch.V = m.V;
  sch.G = m.G;
  sch.num_ctas = m.num_ctas;
  sch.ngran = m.ngran;
  sch.tile_rows = kTileM;
  const uint32_t bg = static_cast<uint32_t>(m.b_off + b);
  const uint64_t k64 = m.row_seeds ? m.row_seeds[bg] : m.seed;
  fs_group_summary *summary = static_cast<fs_group_summary *>(m.summary);

  float best_key = -INFINITY;
  int best_g = -1;
  unsigned long long best_tok = 0ull;
  for (int g = lane; g < m.G; g += 32) {
    const int lo = group_begin(g, m.V, m.G);
    const int hi = group_begin(g + 1, m.V, m.G);
    const int c_first = cta_of(lo, sch);
    const int c_last = cta_of(hi - 1, sch);
    unsigned long long kmax = 0ull;
    float M = -INFINITY, S = 0.f;
    // The group's partials: slots c + g for its CTAs c (2 (c + g) and
    // 2 (c + g) + 1 for CTA pairs c).  Loads go out eight at a time, and the
    // slots are zeroed only after all are read, so the loads overlap.
    const int per_unit = m.pair ? 2 : 1;
    const int nslots = (c_last - c_first + 1) * per_unit;
    auto slot_of = [&](int i) -> size_t {
      const int u = c_first * per_unit + i;
      return m.pair ? 2 * static_cast<size_t>(u / 2 + g) + (u & 1) : static_cast<size_t>(u + g);
    };
    for (int i0 = 0; i0 < nslots; i0 += 8) {
      GroupPartial gp[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (i0 + j < nslots) gp[j] = m.partials[slot_of(i0 + j) * m.B + b];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (i0 + j >= nslots) break;
        kmax = gp[j].key > kmax ? gp[j].key : kmax;
        if (gp[j].m != -INFINITY) {
          if (M == -INFINITY) {
            M = gp[j].m;
            S = gp[j].sum;
          } else {
            const float mx = fmaxf(M, gp[j].m);
            S = S * expf(M - mx) + gp[j].sum * expf(gp[j].m - mx);
            M = mx;
          }
        }
      }
    }
    for (int i = 0; i < nslots; ++i)  // leave the workspace zeroed
      m.partials[slot_of(i) * m.B + b] = GroupPartial{0ull, 0.f, 0.f};
    if (m.gkeys != nullptr) m.gkeys[static_cast<size_t>(g) * m.B + b] = 0ull;  // left zeroed
    const float lse = (M == -INFINITY) ? -INFINITY : M + logf(S);
    if (summary != nullptr) {
      fs_group_summary gs;
      gs.max_score = key_valid(kmax) ? __uint_as_float(key_score_bits(kmax)) : -INFINITY;
      gs.argmax = key_token(kmax);
      gs.lse = lse;
      summary[static_cast<size_t>(b) * m.G + g] = gs;
    }
    if (lse != -INFINITY) {
      const Philox4 ph = philox4x32_10(static_cast<uint32_t>(g) >> 2, bg, m.step, 1u,
                                       static_cast<uint32_t>(k64), static_cast<uint32_t>(k64 >> 32));
      const uint32_t w = (g & 3) == 0 ? ph.w0 : (g & 3) == 1 ? ph.w1 : (g & 3) == 2 ? ph.w2 : ph.w3;
      const float kg = lse + gumbel_from_u32(w);
      if (best_g < 0 || kg > best_key) {  // g rises within a lane: ties keep the smaller g
        best_key = kg;
        best_g = g;
        best_tok = kmax;
      }
    }
  }
  // Warp argmax over (key, group): larger key first, then the smaller group.
  uint64_t packed = best_g < 0 ? 0ull : pack_key(__float_as_uint(best_key), best_g);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, packed, off);
    packed = o > packed ? o : packed;
  }
  const int gwin = key_token(packed);
  const unsigned long long tok =
      __shfl_sync(0xffffffffu, best_tok, gwin < 0 ? 0 : (gwin & 31));
  if (lane == 0 && m.out_idx != nullptr) m.out_idx[b] = gwin < 0 ? -1 : key_token(tok);
}

// Online grouped sampling: Group-Gumbel-Max over summaries [G][B] produced
// one group at a time; the same group noise (tag 1) as the fused grouped path.
__global__ void __launch_bounds__(128)
    merge_summaries_kernel(const fs_group_summary *summaries, int G, int B, uint64_t seed,
                           const uint64_t *row_seeds, uint32_t step, int32_t *out_idx) {
  sm100::grid_dependency_wait();
  const int b = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const uint32_t bg = static_cast<uint32_t>(b);
  const uint64_t k64 = row_seeds ? row_seeds[bg] : seed;
  float best_key = -INFINITY;
  int best_g = -1;
  int best_tok = -1;
  for (int g = lane; g < G; g += 32) {
    const fs_group_summary sm = summaries[static_cast<size_t>(g) * B + b];
    if (sm.lse == -INFINITY || sm.argmax < 0) continue;
    const Philox4 ph = philox4x32_10(static_cast<uint32_t>(g) >> 2, bg, step, 1u,
                                     static_cast<uint32_t>(k64), static_cast<uint32_t>(k64 >> 32));
    const uint32_t w = (g & 3) == 0 ? ph.w0 : (g & 3) == 1 ? ph.w1 : (g & 3) == 2 ? ph.w2 : ph.w3;
    const float kg = sm.lse + gumbel_from_u32(w);
    if (best_g < 0 || kg > best_key) {
      best_key = kg;
      best_g = g;
      best_tok = sm.argmax;
    }
  }
  uint64_t packed = best_g < 0 ? 0ull : pack_key(__float_as_uint(best_key), best_g);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, packed, off);
    packed = o > packed ? o : packed;
  }
  const int gwin = key_token(packed);
  const int tok = __shfl_sync(0xffffffffu, best_tok, gwin < 0 ? 0 : (gwin & 31));
  if (lane == 0) out_idx[b] = gwin < 0 ? -1 : tok;
}

cudaError_t launch_merge_summaries(const void *summaries, int G, int B, uint64_t seed,
                                   const uint64_t *row_seeds, uint32_t step, int32_t *out_idx,
                                   cudaStream_t stream) {
  const int threads = 128;
  const int blocks = (B * 32 + threads - 1) / threads;
  return launch_dependent(merge_summaries_kernel, dim3(blocks), dim3(threads), stream,
                          static_cast<const fs_group_summary *>(summaries), G, B, seed, row_seeds,
                          step, out_idx);
}

cudaError_t launch_group_merge(const MergeParams &m, cudaStream_t stream) {
  const int threads = 128;
  const int blocks = (m.B * 32 + threads - 1) / threads;
  return launch_dependent(group_merge_kernel, dim3(blocks), dim3(threads), stream, m);
}

// ---------------------------------------------------------------------------
// Unfused mode, kernel 2: temperature, mask, noise and argmax over fp32
// logits [B][V].  Each thread takes four consecutive tokens (one Philox
// call); blocks publish a packed max per row with atomicMax and the last
// block decodes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) sample_logits_kernel(const SampleLogitsParams s) {
  sm100::grid_dependency_wait();  // the logits
  const int b = blockIdx.y;
  const uint32_t bg = static_cast<uint32_t>(s.b_off + b);
  const uint64_t k64 = s.row_seeds ? s.row_seeds[bg] : s.seed;
  const float *row = s.logits + static_cast<size_t>(b) * s.V;
  const int nquads = (s.V + 3) / 4;
  const bool vec = (s.V & 3) == 0;
  uint64_t best = 0ull;
  for (int qd = blockIdx.x * blockDim.x + threadIdx.x; qd < nquads; qd += gridDim.x * blockDim.x) {
    const Philox4 ph = philox4x32_10(static_cast<uint32_t>(qd), bg, s.step, 0u,
                                     static_cast<uint32_t>(k64), static_cast<uint32_t>(k64 >> 32));
    const uint32_t w[4] = {ph.w0, ph.w1, ph.w2, ph.w3};
    float l[4];
    const int v0 = 4 * qd;
    if (vec) {
      const float4 l4 = *reinterpret_cast<const float4 *>(row + v0);
      l[0] = l4.x;
      l[1] = l4.y;
      l[2] = l4.z;
      l[3] = l4.w;
    } else {
#pragma unroll
      for (int m = 0; m < 4; ++m) l[m] = (v0 + m < s.V) ? row[v0 + m] : 0.f;
    }
    uint32_t mword = 0xFFFFFFFFu;
    if (s.mask) mword = s.mask[static_cast<size_t>(bg) * s.mask_words + (v0 >> 5)];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int v = v0 + m;
      const bool ok = v < s.V && ((mword >> (v & 31)) & 1u);
      const float sc = fmaf(l[m], s.inv_temp, gumbel_from_u32(w[m]));  // as the fused kernel
      const uint64_t k = ok ? pack_key(__float_as_uint(sc), v) : 0ull;
      best = k > best ? k : best;
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
    best = o > best ? o : best;
  }
  __shared__ uint64_t warp_best[8];
  __shared__ int is_last;
  if ((threadIdx.x & 31) == 0) warp_best[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t r = 0ull;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) r = warp_best[i] > r ? warp_best[i] : r;
    if (key_valid(r)) atomicMax(s.keys + b, static_cast<unsigned long long>(r));
    __threadfence();
    const unsigned total = gridDim.x * gridDim.y;
    is_last = (atomicAdd(s.ticket, 1u) == total - 1) ? 1 : 0;
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    for (int r = threadIdx.x; r < s.B; r += blockDim.x)
      s.out_idx[r] = key_token(atomicExch(s.keys + r, 0ull));
    if (threadIdx.x == 0) atomicExch(s.ticket, 0u);
  }
}

cudaError_t launch_sample_logits(const SampleLogitsParams &s, cudaStream_t stream) {
  const int threads = 256;
  const int nquads = (s.V + 3) / 4;
  int per_row = (nquads + threads - 1) / threads;
  const int target = (4 * s.num_sms + s.B - 1) / s.B;  // about four blocks per SM in total
  if (per_row > target) per_row = target;
  if (per_row < 1) per_row = 1;
  return launch_dependent(sample_logits_kernel, dim3(per_row, s.B), dim3(threads), stream, s);
}

// ---------------------------------------------------------------------------
// Top-k sampling over fp32 logits [B][V] (readus.org page, "Top-K and
// masking": a prefilter isolates the candidates, exact Gumbel-max runs on
// them).  An exact radix select finds each row's k-th largest
// order-preserving key among the allowed logits, over bits 31-21, 20-10 and
// 9-0; the candidates -- keys above it, and as many keys equal to it as k
// allows, in index order -- then get their noise and the Gumbel-max.  Each
// row is split over P blocks (P x rows ~ two blocks per SM), one launch per
// pass: three histogram passes into per-row global histograms, then the
// candidate pass, whose last block per row writes the token and re-zeroes
// the row's scratch.
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkItems = 8;      // consecutive elements per thread per iteration
constexpr int kTopkBins = 2048;
constexpr int kTopkSubHists = 4;   // warp-interleaved copies of the shared histogram
constexpr int kTopkMinSlice = kTopkThreads * kTopkItems;

// Per-launch scratch offsets for `rows` rows split over P blocks each.
struct TopkLayout {
  size_t hist0, hist1, hist2, hist2blk, rowkey, ticket, bytes;
};
static TopkLayout topk_layout(int rows, int P) {
  TopkLayout l;
  size_t o = 0;
  l.hist0 = o;    o += static_cast<size_t>(rows) * kTopkBins * 4;
  l.hist1 = o;    o += static_cast<size_t>(rows) * kTopkBins * 4;
  l.hist2 = o;    o += static_cast<size_t>(rows) * 1024 * 4;
  l.hist2blk = o; o += static_cast<size_t>(rows) * P * 1024 * 4;
  l.rowkey = o;   o += static_cast<size_t>(rows) * 8;
  l.ticket = o;   o += static_cast<size_t>(rows) * 4;
  l.bytes = (o + 255) / 256 * 256;
  return l;
}

// Blocks per row: as many as keep the grid within one wave of two
// 1024-thread blocks per SM, each with at least kTopkMinSlice tokens.
static int topk_blocks_per_row(int rows, int V, int num_sms) {
  const int want = 2 * num_sms / rows;
  const int most = (V + kTopkMinSlice - 1) / kTopkMinSlice;
  return want < 1 ? 1 : (want > most ? most : want);
}

size_t topk_scratch_bytes(int rows, int V, int num_sms) {
  return topk_layout(rows, topk_blocks_per_row(rows, V, num_sms)).bytes;
}

struct TopkArgs {
  SampleLogitsParams s;
  int K, P, slice;
  int *hist0, *hist1, *hist2, *hist2blk;
  unsigned long long *rowkey;
  unsigned int *ticket;
};

// Block-wide exclusive scan of one int per thread (1024 threads); returns the
// thread's prefix and writes the total to *total.
__device__ __forceinline__ int block_exclusive_scan(int x, int *warp_sums, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    warp_sums[lane] = wi - w;  // exclusive prefix of the warp totals
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - x;
  __syncthreads();
  return r;
}

struct TopkShared {
  int hist[kTopkSubHists * kTopkBins];
  int warp_sums[32];
  int digit, above, total;
  unsigned long long warp_best[32];
};

// The digit of a global histogram row (nb = 2048 or 1024 bins) that holds the
// k-th largest key (1-based): sets sh.digit and sh.above (keys in higher
// bins).  With total_out, also the histogram's total.
__device__ void topk_select_digit(const int *h, int nb, int k, TopkShared &sh, int *total_out) {
  int c_hi, c_lo, hi_bin, lo_bin;
  if (nb == kTopkBins) {
    const int t = kTopkThreads - 1 - threadIdx.x;  // thread 0 holds the two top bins
    hi_bin = 2 * t + 1;
    lo_bin = 2 * t;
    c_hi = __ldcg(h + hi_bin);
    c_lo = __ldcg(h + lo_bin);
  } else {
    hi_bin = nb - 1 - threadIdx.x;
    lo_bin = -1;
    c_hi = __ldcg(h + hi_bin);
    c_lo = 0;
  }
  const int above = block_exclusive_scan(c_hi + c_lo, sh.warp_sums, &sh.total);
  if (total_out) *total_out = sh.total;
  if (above < k && above + c_hi >= k) {
    sh.digit = hi_bin;
    sh.above = above;
  } else if (lo_bin >= 0 && above + c_hi < k && above + c_hi + c_lo >= k) {
    sh.digit = lo_bin;
    sh.above = above + c_hi;
  }
  __syncthreads();
}

// Loads this thread's kTopkItems consecutive logits starting at v0 (below
// hi) and their order-preserving keys; ok[i] is false past hi or for a
// masked token.
__device__ __forceinline__ void topk_load(const SampleLogitsParams &s, const float *row,
                                          uint32_t bg, int v0, int hi, bool vec,
                                          float (&l)[kTopkItems], uint32_t (&key)[kTopkItems],
                                          bool (&ok)[kTopkItems]) {
  if (vec && v0 + kTopkItems <= hi) {
    const float4 a = *reinterpret_cast<const float4 *>(row + v0);
    const float4 c = *reinterpret_cast<const float4 *>(row + v0 + 4);
    l[0] = a.x; l[1] = a.y; l[2] = a.z; l[3] = a.w;
    l[4] = c.x; l[5] = c.y; l[6] = c.z; l[7] = c.w;
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i) ok[i] = true;
  } else {
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i) {
      ok[i] = v0 + i < hi;
      l[i] = ok[i] ? row[v0 + i] : 0.f;
    }
  }
  uint32_t mword = 0xFFFFFFFFu;
  if (s.mask != nullptr && v0 < hi)   // 8 consecutive tokens from a multiple of 8 share one word
    mword = s.mask[static_cast<size_t>(bg) * s.mask_words + (v0 >> 5)];
#pragma unroll
  for (int i = 0; i < kTopkItems; ++i) {
    ok[i] = ok[i] && ((mword >> ((v0 + i) & 31)) & 1u);
    key[i] = order_bits(__float_as_uint(l[i]));
  }
}

// The selection state before pass `pass`: the key prefix found so far, its
// mask, the rank still to find among keys matching it, and whether every
// allowed token is a candidate (k >= allowed tokens).
struct TopkState {
  uint32_t prefix, pmask;
  int k_rem;
  bool all_allowed;
};

__device__ TopkState topk_state(const TopkArgs &a, int b, int passes, TopkShared &sh) {
  TopkState st{0u, 0u, a.K, false};
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  const int *hists[3] = {a.hist0, a.hist1, a.hist2};
  for (int pass = 0; pass < passes; ++pass) {
    const int nb = 1 << widths[pass];
    int total = 0;
    topk_select_digit(hists[pass] + static_cast<size_t>(b) * (pass < 2 ? kTopkBins : 1024), nb,
                      st.k_rem, sh, pass == 0 ? &total : nullptr);
    if (pass == 0 && total <= a.K) {
      st.all_allowed = true;
      return st;
    }
    st.prefix |= static_cast<uint32_t>(sh.digit) << shifts[pass];
    st.pmask |= static_cast<uint32_t>(nb - 1) << shifts[pass];
    st.k_rem -= sh.above;
    __syncthreads();
  }
  return st;
}

// Histogram pass `PASS` (0, 1, 2) of block (p, b) over its slice.
template <int PASS>
__global__ void __launch_bounds__(kTopkThreads) topk_hist_kernel(const TopkArgs a) {
  __shared__ TopkShared sh;
  sm100::grid_dependency_wait();  // the logits, or the previous pass's histograms
  const int p = blockIdx.x, b = blockIdx.y;
  const SampleLogitsParams &s = a.s;
  const uint32_t bg = static_cast<uint32_t>(s.b_off + b);
  const float *row = s.logits + static_cast<size_t>(b) * s.V;
  const int lo = p * a.slice, hi = imin(s.V, lo + a.slice);
  const bool vec = (s.V & 3) == 0;
  const TopkState st = topk_state(a, b, PASS, sh);
  if (st.all_allowed) return;
  constexpr int kShift = PASS == 0 ? 21 : (PASS == 1 ? 10 : 0);
  constexpr uint32_t kDMask = PASS == 2 ? 1023u : 2047u;
  constexpr int kBins = PASS == 2 ? 1024 : kTopkBins;
  for (int i = threadIdx.x; i < kTopkSubHists * kBins; i += kTopkThreads) sh.hist[i] = 0;
  __syncthreads();
  int *my_hist = sh.hist + ((threadIdx.x >> 5) & (kTopkSubHists - 1)) * kBins;
  for (int base = lo; base < hi; base += kTopkThreads * kTopkItems) {
    float l[kTopkItems];
    uint32_t key[kTopkItems];
    bool ok[kTopkItems];
    topk_load(s, row, bg, base + threadIdx.x * kTopkItems, hi, vec, l, key, ok);
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i)
      if (ok[i] && (key[i] & st.pmask) == st.prefix)
        atomicAdd(&my_hist[(key[i] >> kShift) & kDMask], 1);
  }
  __syncthreads();
  int *gh = (PASS == 0 ? a.hist0 : PASS == 1 ? a.hist1 : a.hist2) +
            static_cast<size_t>(b) * kBins;
  for (int i = threadIdx.x; i < kBins; i += kTopkThreads) {
    int c = 0;
#pragma unroll
    for (int h = 0; h < kTopkSubHists; ++h) c += sh.hist[h * kBins + i];
    if (c) atomicAdd(gh + i, c);
    if (PASS == 2) a.hist2blk[(static_cast<size_t>(b) * a.P + p) * 1024 + i] = c;
  }
}

// Candidate pass of block (p, b): Gumbel-max over the slice's candidates; the
// last block of the row writes its token and re-zeroes the row's scratch.
__global__ void __launch_bounds__(kTopkThreads) topk_final_kernel(const TopkArgs a) {
  __shared__ TopkShared sh;
  __shared__ int last_block;
  sm100::grid_dependency_wait();  // the histograms
  const int p = blockIdx.x, b = blockIdx.y;
  const SampleLogitsParams &s = a.s;
  const uint32_t bg = static_cast<uint32_t>(s.b_off + b);
  const float *row = s.logits + static_cast<size_t>(b) * s.V;
  const int lo = p * a.slice, hi = imin(s.V, lo + a.slice);
  const bool vec = (s.V & 3) == 0;
  const int lane = threadIdx.x & 31;
  const TopkState st = topk_state(a, b, 3, sh);
  // Keys equal to the k-th largest: the first k_rem of them, in index order,
  // are candidates; blocks before this one hold `before` of them.
  int take = 0, n_eq = 0;
  if (!st.all_allowed) {
    const int digit = static_cast<int>(st.prefix & 1023u);
    const int *hb = a.hist2blk + static_cast<size_t>(b) * a.P * 1024 + digit;
    int before = 0;
    for (int q = 0; q < p; ++q) before += __ldcg(hb + static_cast<size_t>(q) * 1024);
    n_eq = __ldcg(hb + static_cast<size_t>(p) * 1024);
    take = imin(imax(st.k_rem - before, 0), n_eq);
  }
  // Ranking the equal keys in index order is needed only when some but not
  // all of this slice's equal keys are candidates (block-uniform).
  const bool rank_ties = take > 0 && take < n_eq;
  const uint64_t k64 = s.row_seeds ? s.row_seeds[bg] : s.seed;
  uint64_t best = 0ull;
  int eq_seen = 0;
  for (int base = lo; base < hi; base += kTopkThreads * kTopkItems) {
    const int v0 = base + threadIdx.x * kTopkItems;
    float l[kTopkItems];
    uint32_t key[kTopkItems];
    bool ok[kTopkItems];
    topk_load(s, row, bg, v0, hi, vec, l, key, ok);
    int r = 0;
    if (rank_ties) {
      int n_eq_mine = 0;
#pragma unroll
      for (int i = 0; i < kTopkItems; ++i) n_eq_mine += (ok[i] && key[i] == st.prefix) ? 1 : 0;
      r = eq_seen + block_exclusive_scan(n_eq_mine, sh.warp_sums, &sh.total);
      eq_seen += sh.total;
    }
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i) {
      if (!ok[i]) continue;
      bool cand = st.all_allowed || key[i] > st.prefix;
      if (!st.all_allowed && key[i] == st.prefix) {
        cand = rank_ties ? r < take : take > 0;
        ++r;
      }
      if (cand) {
        const int v = v0 + i;
        const Philox4 ph = philox4x32_10(static_cast<uint32_t>(v) >> 2, bg, s.step, 0u,
                                         static_cast<uint32_t>(k64),
                                         static_cast<uint32_t>(k64 >> 32));
        const uint32_t w =
            (v & 3) == 0 ? ph.w0 : (v & 3) == 1 ? ph.w1 : (v & 3) == 2 ? ph.w2 : ph.w3;
        const float sc = fmaf(l[i], s.inv_temp, gumbel_from_u32(w));
        const uint64_t k = pack_key(__float_as_uint(sc), v);
        best = k > best ? k : best;
      }
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
    best = o > best ? o : best;
  }
  if (lane == 0) sh.warp_best[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t r = 0ull;
    for (int i = 0; i < kTopkThreads / 32; ++i) r = sh.warp_best[i] > r ? sh.warp_best[i] : r;
    if (r) atomicMax(a.rowkey + b, static_cast<unsigned long long>(r));
    __threadfence();
    last_block = atomicAdd(a.ticket + b, 1u) == static_cast<unsigned>(a.P - 1);
  }
  __syncthreads();
  if (last_block) {
    __threadfence();
    if (threadIdx.x == 0) {
      const unsigned long long kb = atomicExch(a.rowkey + b, 0ull);
      s.out_idx[b] = key_token(kb);
      a.ticket[b] = 0u;
    }
    // every block of the row has read the histograms before taking its ticket
    for (int i = threadIdx.x; i < kTopkBins; i += kTopkThreads) {
      a.hist0[static_cast<size_t>(b) * kTopkBins + i] = 0;
      a.hist1[static_cast<size_t>(b) * kTopkBins + i] = 0;
    }
    for (int i = threadIdx.x; i < 1024; i += kTopkThreads) a.hist2[static_cast<size_t>(b) * 1024 + i] = 0;
    for (int i = threadIdx.x; i < a.P * 1024; i += kTopkThreads)
      a.hist2blk[static_cast<size_t>(b) * a.P * 1024 + i] = 0;
  }
}

cudaError_t launch_topk_sample(const SampleLogitsParams &s, int K, void *scratch,
                               cudaStream_t stream) {
  const int P = topk_blocks_per_row(s.B, s.V, s.num_sms);
  const TopkLayout lay = topk_layout(s.B, P);
  char *base = static_cast<char *>(scratch);
  TopkArgs a;
  a.s = s;
  a.K = K;
  a.P = P;
  a.slice = ((s.V + P - 1) / P + kTopkItems - 1) / kTopkItems * kTopkItems;
  a.hist0 = reinterpret_cast<int *>(base + lay.hist0);
  a.hist1 = reinterpret_cast<int *>(base + lay.hist1);
  a.hist2 = reinterpret_cast<int *>(base + lay.hist2);
  a.hist2blk = reinterpret_cast<int *>(base + lay.hist2blk);
  a.rowkey = reinterpret_cast<unsigned long long *>(base + lay.rowkey);
  a.ticket = reinterpret_cast<unsigned int *>(base + lay.ticket);
  const dim3 grid(P, s.B), block(kTopkThreads);
  cudaError_t e;
  if ((e = launch_dependent(topk_hist_kernel<0>, grid, block, stream, a)) != cudaSuccess) return e;
  if ((e = launch_dependent(topk_hist_kernel<1>, grid, block, stream, a)) != cudaSuccess) return e;
  if ((e = launch_dependent(topk_hist_kernel<2>, grid, block, stream, a)) != cudaSuccess) return e;
  return launch_dependent(topk_final_kernel, grid, block, stream, a);
}

// ---------------------------------------------------------------------------
// Vocabulary shards: tokens from the reduced keys.
// ---------------------------------------------------------------------------
__global__ void keys_to_tokens_kernel(const long long *keys, int B, int32_t *out_idx) {
  sm100::grid_dependency_wait();  // the reduced keys
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) out_idx[b] = key_token(static_cast<uint64_t>(keys[b]) ^ 0x8000000000000000ull);
}

cudaError_t launch_keys_to_tokens(const long long *keys, int B, int32_t *out_idx,
                                  cudaStream_t stream) {
  return launch_dependent(keys_to_tokens_kernel, dim3((B + 255) / 256), dim3(256), stream, keys, B,
                          out_idx);
}

// ---------------------------------------------------------------------------
// Test kernels
// ---------------------------------------------------------------------------
__global__ void philox_test_kernel(const uint32_t *ctr, const uint32_t *key, uint32_t *out,
                                   int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const Philox4 ph = philox4x32_10(ctr[4 * i], ctr[4 * i + 1], ctr[4 * i + 2], ctr[4 * i + 3],
                                     key[2 * i], key[2 * i + 1]);
    out[4 * i] = ph.w0;
    out[4 * i + 1] = ph.w1;
    out[4 * i + 2] = ph.w2;
    out[4 * i + 3] = ph.w3;
  }
}

__global__ void gumbel_test_kernel(const uint32_t *r, float *g, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    g[i] = gumbel_from_u32(r[i]);
}

static int test_grid(int64_t n) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return blocks < 1 ? 1 : static_cast<int>(blocks);
}

cudaError_t launch_philox_test(const uint32_t *ctr, const uint32_t *key, uint32_t *out, int64_t n,
                               cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  philox_test_kernel<<<test_grid(n), 256, 0, stream>>>(ctr, key, out, n);
  return cudaGetLastError();
}

cudaError_t launch_gumbel_test(const uint32_t *r, float *g, int64_t n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  gumbel_test_kernel<<<test_grid(n), 256, 0, stream>>>(r, g, n);
  return cudaGetLastError();
}

}  // namespace fmms
