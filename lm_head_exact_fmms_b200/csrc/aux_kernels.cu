// aux_kernels.cu -- the small kernels around the fused one:
//  * the Group-Gumbel-Max merge of per-(segment, row) partials (readus.org
//    page, "Group Gumbel Max": pick a group with Gumbel noise on the group
//    log-masses, then take the sample inside the winning group);
//  * the second kernel of the unfused mode, sampling from fp32 logits in HBM;
//  * the bounded wait of the tensor-parallel exchange;
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
static cudaError_t launch_dependent_smem(void (*kern)(KArgs...), dim3 grid, dim3 block,
                                         size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block,
                                    cudaStream_t stream, Args... args) {
  return launch_dependent_smem(kern, grid, block, 0, stream, args...);
}

// ---------------------------------------------------------------------------
// Group merge: one warp per row; lanes stride over the groups, or with at
// most four groups teams of lanes share each group's partials.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) group_merge_kernel(const MergeParams m) {
  // The kernel after this one may start launching now: a fused sampling
  // kernel launched as a programmatic dependent streams W meanwhile and
  // waits for this grid to complete before it loads H or touches the
  // workspace or the outputs this grid writes.
  sm100::launch_dependents();
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
  const uint64_t k64 =
      (m.row_seeds && FS_IN_BOUNDS(m.err, bg, m.rows_total)) ? m.row_seeds[bg] : m.seed;
  fs_group_summary *summary = static_cast<fs_group_summary *>(m.summary);

  float best_key = -INFINITY;
  int best_g = -1;
  unsigned long long best_tok = 0ull;
  // With few groups a team of lanes shares one group's partials (a group of
  // a single-group call spans every CTA: 148 slots a row), else each lane
  // takes whole groups.  Teams are aligned runs of `team` lanes.
  const int team = m.G == 1 ? 32 : m.G == 2 ? 16 : m.G <= 4 ? 8 : 1;
  const int member = lane & (team - 1);
  const int nteams = 32 / team;
  for (int g0 = 0; g0 < m.G; g0 += nteams) {  // warp-uniform
    const int g = g0 + lane / team;
    const bool gok = g < m.G;
    unsigned long long kmax = 0ull;
    float M = -INFINITY, S = 0.f;
    // The group's partials: slots c + g for its CTAs c (2 (c + g) and
    // 2 (c + g) + 1 for CTA pairs c).  A member takes slots member,
    // member + team, ...; loads go out eight at a time, and the slots are
    // zeroed only after all are read, so the loads overlap.
    int c_first = 0, nslots = 0;
    const int per_unit = m.pair ? 2 : 1;
    if (gok) {
      const int lo = group_begin(g, m.V, m.G);
      const int hi = group_begin(g + 1, m.V, m.G);
      c_first = cta_of(lo, sch);
      nslots = (cta_of(hi - 1, sch) - c_first + 1) * per_unit;
    }
    auto slot_of = [&](int i) -> size_t {
      const int u = c_first * per_unit + i;
      return m.pair ? 2 * static_cast<size_t>(u / 2 + g) + (u & 1) : static_cast<size_t>(u + g);
    };
    for (int i0 = member; i0 < nslots; i0 += 8 * team) {
      GroupPartial gp[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * team;
        gp[j] = GroupPartial{0ull, -INFINITY, 0.f};
        if (i < nslots &&
            FS_IN_BOUNDS(m.err, static_cast<long long>(slot_of(i)) * m.B + b, m.partials_cap))
          gp[j] = m.partials[slot_of(i) * m.B + b];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (i0 + j * team >= nslots) break;
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
    for (int i = member; i < nslots; i += team)  // leave the workspace zeroed
      if (FS_IN_BOUNDS(m.err, static_cast<long long>(slot_of(i)) * m.B + b, m.partials_cap))
        m.partials[slot_of(i) * m.B + b] = GroupPartial{0ull, 0.f, 0.f};
    // Team reduction: the maximum key and the merged (max, sum) pair.
    for (int off = team / 2; off >= 1; off >>= 1) {
      const unsigned long long ko = __shfl_xor_sync(0xffffffffu, kmax, off);
      const float Mo = __shfl_xor_sync(0xffffffffu, M, off);
      const float So = __shfl_xor_sync(0xffffffffu, S, off);
      kmax = ko > kmax ? ko : kmax;
      if (Mo != -INFINITY) {
        if (M == -INFINITY) {
          M = Mo;
          S = So;
        } else {
          const float mx = fmaxf(M, Mo);
          S = S * expf(M - mx) + So * expf(Mo - mx);
          M = mx;
        }
      }
    }
    if (!gok || member != 0) continue;
    if (m.gkeys != nullptr &&
        FS_IN_BOUNDS(m.err, static_cast<long long>(g) * m.B + b, m.gkeys_cap))
      m.gkeys[static_cast<size_t>(g) * m.B + b] = 0ull;  // left zeroed
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
  // group g was taken by the first lane of team g mod nteams
  const unsigned long long tok =
      __shfl_sync(0xffffffffu, best_tok, gwin < 0 ? 0 : (gwin % nteams) * team);
  if (lane == 0 && m.out_idx != nullptr) m.out_idx[b] = gwin < 0 ? -1 : key_token(tok);
}

// Online grouped sampling: Group-Gumbel-Max over summaries [G][B] produced
// one group at a time; the same group noise (tag 1) as the fused grouped path.
__global__ void __launch_bounds__(128)
    merge_summaries_kernel(const fs_group_summary *summaries, int G, int B, uint64_t seed,
                           const uint64_t *row_seeds, uint32_t step, int32_t *out_idx) {
  // The kernel after this one may start launching now: a fused sampling
  // kernel launched as a programmatic dependent streams W meanwhile and
  // waits for this grid to complete before it loads H or touches the
  // workspace or the outputs this grid writes.
  sm100::launch_dependents();
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
  // The kernel after this one may start launching now: a fused sampling
  // kernel launched as a programmatic dependent streams W meanwhile and
  // waits for this grid to complete before it loads H or touches the
  // workspace or the outputs this grid writes.
  sm100::launch_dependents();
  sm100::grid_dependency_wait();  // the logits
  const int b = blockIdx.y;
  const uint32_t bg = static_cast<uint32_t>(s.b_off + b);
  const uint64_t k64 =
      (s.row_seeds && FS_IN_BOUNDS(s.err, bg, s.rows_total)) ? s.row_seeds[bg] : s.seed;
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
    if (s.mask && FS_IN_BOUNDS(s.err, bg, s.rows_total) &&
        FS_IN_BOUNDS(s.err, v0 >> 5, s.mask_words))
      mword = s.mask[static_cast<size_t>(bg) * s.mask_words + (v0 >> 5)];
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
    if (key_valid(r) && FS_IN_BOUNDS(s.err, b, kMaxBN))
      atomicMax(s.keys + b, static_cast<unsigned long long>(r));
    __threadfence();
    const unsigned total = gridDim.x * gridDim.y;
    is_last = (atomicAdd(s.ticket, 1u) == total - 1) ? 1 : 0;
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    for (int r = threadIdx.x; r < s.B; r += blockDim.x)
      if (FS_IN_BOUNDS(s.err, r, kMaxBN)) s.out_idx[r] = key_token(atomicExch(s.keys + r, 0ull));
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
// them).  The candidates of a row are its K allowed tokens with the largest
// logits, ties toward the smaller index.  Two launches:
//   1. topk_local_kernel: each row is split over P blocks (P x rows at most
//      one block per SM, so the grid is one wave).  A block finds a key
//      threshold at or below its slice's K-th largest allowed key (or 0 when
//      the slice has at most K) whose passing keys fit its capacity -- read
//      off a histogram of a sample and verified by the extraction pass, else
//      set by exact shared-memory radix histograms of the slice, down to the
//      exact key with its tied tokens ranked in token order -- and writes the
//      passing (key, token) pairs and the threshold.  The row's K-th largest
//      key is at least every block's threshold, so the union of the lists
//      holds the row's top K and every token tied with the row's K-th key.
//   2. topk_row_kernel: one block per row keeps the candidates at or above
//      the largest block threshold, selects the exact top K among them (one
//      radix level, then direct ranks; larger sets take three radix levels
//      and a radix select on the token for a split tie), draws the noise of
//      the selected tokens and writes the Gumbel-max token.
// Nothing carries over between calls: the list lengths and thresholds are
// written, not accumulated.
// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkItems = 16;     // consecutive elements per thread per iteration (4 x 16 B)
constexpr int kTopkBins = 2048;
constexpr int kTopkSubHists = 4;   // warp-interleaved copies of the shared histogram
constexpr int kTopkMinSlice = kTopkThreads * kTopkItems;
constexpr int kTopkMinCap = 2048;  // candidate capacity per block, at least K
constexpr int kTopkMaxP = 512;
constexpr int kTopkRowCap = 8192;  // candidates a row's select block keeps in shared memory
constexpr int kTopkRowSmall = 256; // at most this many left after one radix level: rank them

struct TopkGeom {
  int P, slice, cap;
};
static TopkGeom topk_geom(int rows, int V, int K, int num_sms) {
  TopkGeom g;
  const int want = num_sms / rows;  // one wave: a 1024-thread block fills an SM's registers
  const int most = (V + kTopkMinSlice - 1) / kTopkMinSlice;
  g.P = want < 1 ? 1 : (want > most ? most : want);
  if (g.P > kTopkMaxP) g.P = kTopkMaxP;
  g.slice = ((V + g.P - 1) / g.P + kTopkItems - 1) / kTopkItems * kTopkItems;
  g.cap = K > kTopkMinCap ? K : kTopkMinCap;
  if (g.cap > g.slice) g.cap = g.slice;
  return g;
}

size_t topk_scratch_bytes(int rows, int V, int K, int num_sms) {
  const TopkGeom g = topk_geom(rows, V, K, num_sms);
  const size_t lists = static_cast<size_t>(rows) * g.P * g.cap * 8;
  const size_t counts = static_cast<size_t>(rows) * g.P * 8;  // lengths and thresholds
  return (lists + counts + 255) / 256 * 256;
}

struct TopkArgs {
  SampleLogitsParams s;
  int K, P, slice, cap;
  unsigned long long *cand;  // [rows][P][cap]: (key << 32) | token
  int *cnt;                  // [rows][P]: list lengths
  unsigned int *thr;         // [rows][P]: each block's key threshold (0: every allowed key)
};

// Block-wide exclusive scan of one int per thread (1024 threads); returns the
// thread's prefix and writes the total to *total, which must be in shared
// memory (one thread writes it, every thread may read it after the call).
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

// The digit of a shared histogram (nb = 2048 or 1024 bins, in sh.hist) that
// holds the k-th largest key (1-based): returns it and its count, and sets
// *above to the keys in higher bins.  *total gets the histogram's total; when
// it is below k the digit is 0 and the other results are meaningless.
__device__ int topk_select_digit(int nb, int k, TopkShared &sh, int *above, int *count,
                                 int *total) {
  if (threadIdx.x == 0) {  // ordered before the writes below by the scan's barriers
    sh.digit = 0;
    sh.above = 0;
  }
  int c_hi, c_lo, hi_bin, lo_bin;
  if (nb == kTopkBins) {
    const int t = kTopkThreads - 1 - threadIdx.x;  // thread 0 holds the two top bins
    hi_bin = 2 * t + 1;
    lo_bin = 2 * t;
    c_hi = sh.hist[hi_bin];
    c_lo = sh.hist[lo_bin];
  } else {
    hi_bin = nb - 1 - threadIdx.x;
    lo_bin = -1;
    c_hi = sh.hist[hi_bin];
    c_lo = 0;
  }
  const int ab = block_exclusive_scan(c_hi + c_lo, sh.warp_sums, &sh.total);
  if (ab < k && ab + c_hi >= k) {
    sh.digit = hi_bin;
    sh.above = ab;
  } else if (lo_bin >= 0 && ab + c_hi < k && ab + c_hi + c_lo >= k) {
    sh.digit = lo_bin;
    sh.above = ab + c_hi;
  }
  __syncthreads();
  const int d = sh.digit;
  *above = sh.above;
  *count = sh.hist[d];
  *total = sh.total;
  __syncthreads();  // the caller may rebuild sh.hist next
  return d;
}

// Loads this thread's kTopkItems consecutive logits starting at v0 (below
// hi; four 16-byte loads in flight when the row allows) as order-preserving
// keys; bit i of the result is set for an in-range, allowed token v0 + i.
__device__ __forceinline__ uint32_t topk_load(const SampleLogitsParams &s, const float *row,
                                              uint32_t bg, int v0, int hi, bool vec,
                                              uint32_t (&key)[kTopkItems]) {
  uint32_t okm;
  if (vec && v0 + kTopkItems <= hi) {
    const float4 *src = reinterpret_cast<const float4 *>(row + v0);
    float4 q[kTopkItems / 4];
#pragma unroll
    for (int j = 0; j < kTopkItems / 4; ++j) q[j] = src[j];
#pragma unroll
    for (int j = 0; j < kTopkItems / 4; ++j) {
      key[4 * j + 0] = __float_as_uint(q[j].x);
      key[4 * j + 1] = __float_as_uint(q[j].y);
      key[4 * j + 2] = __float_as_uint(q[j].z);
      key[4 * j + 3] = __float_as_uint(q[j].w);
    }
    okm = (1u << kTopkItems) - 1u;
  } else {
    okm = 0u;
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i) {
      const bool in = v0 + i < hi;
      key[i] = in ? __float_as_uint(row[v0 + i]) : 0u;
      okm |= in ? (1u << i) : 0u;
    }
  }
  if (s.mask != nullptr && v0 < hi)  // 16 tokens from a multiple of 16 lie in one mask word
    if (FS_IN_BOUNDS(s.err, bg, s.rows_total) && FS_IN_BOUNDS(s.err, v0 >> 5, s.mask_words))
      okm &= s.mask[static_cast<size_t>(bg) * s.mask_words + (v0 >> 5)] >> (v0 & 31);
#pragma unroll
  for (int i = 0; i < kTopkItems; ++i) key[i] = order_bits(key[i]);
  return okm;
}

// Histogram, in sh.hist[0, nb), of digit (key >> shift) & (nb - 1) over the
// allowed keys of [lo, hi) with (key & pmask) == prefix.
__device__ void topk_slice_hist(const SampleLogitsParams &s, const float *row, uint32_t bg,
                                int lo, int hi, bool vec, uint32_t prefix, uint32_t pmask,
                                int shift, int nb, TopkShared &sh) {
  for (int i = threadIdx.x; i < kTopkSubHists * nb; i += kTopkThreads) sh.hist[i] = 0;
  __syncthreads();
  int *my_hist = sh.hist + ((threadIdx.x >> 5) & (kTopkSubHists - 1)) * nb;
  const uint32_t dmask = static_cast<uint32_t>(nb - 1);
  for (int base = lo; base < hi; base += kTopkThreads * kTopkItems) {
    uint32_t key[kTopkItems];
    const uint32_t okm = topk_load(s, row, bg, base + threadIdx.x * kTopkItems, hi, vec, key);
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i)
      if (((okm >> i) & 1u) && (key[i] & pmask) == prefix)
        atomicAdd(&my_hist[(key[i] >> shift) & dmask], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nb; i += kTopkThreads) {
    int c = 0;
#pragma unroll
    for (int h = 0; h < kTopkSubHists; ++h) c += sh.hist[h * nb + i];
    sh.hist[i] = c;  // thread i alone reads and writes bin i of every copy
  }
  __syncthreads();
}

// Appends the allowed keys of [lo, hi) that pass the threshold -- keys >=
// lo_key, or in exact mode keys > lo_key and the first `take` keys equal to
// it in token order -- to `out` (capacity cap; *n_out counts every passing
// key, stored or not) and counts the allowed keys into *n_ok.
__device__ void topk_extract(const SampleLogitsParams &s, const float *row, uint32_t bg, int lo,
                             int hi, bool vec, uint32_t lo_key, bool exact, int take,
                             unsigned long long *out, int cap, int *n_out, int *n_ok,
                             TopkShared &sh) {
  const int lane = threadIdx.x & 31;
  int eq_seen = 0, ok_mine = 0;
  for (int base = lo; base < hi; base += kTopkThreads * kTopkItems) {
    const int v0 = base + threadIdx.x * kTopkItems;
    uint32_t key[kTopkItems];
    const uint32_t okm = topk_load(s, row, bg, v0, hi, vec, key);
    int r = 0;
    if (exact) {  // block-uniform: rank the tied keys in token order
      int n_eq = 0;
#pragma unroll
      for (int i = 0; i < kTopkItems; ++i) n_eq += (((okm >> i) & 1u) && key[i] == lo_key) ? 1 : 0;
      r = eq_seen + block_exclusive_scan(n_eq, sh.warp_sums, &sh.total);
      eq_seen += sh.total;
    }
    uint32_t sel = 0u;
    ok_mine += __popc(okm);
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i) {
      if (!((okm >> i) & 1u)) continue;
      bool c;
      if (exact) {
        c = key[i] > lo_key;
        if (key[i] == lo_key) c = r++ < take;
      } else {
        c = key[i] >= lo_key;
      }
      if (c) sel |= 1u << i;
    }
    // Warp-aggregated append: one shared-memory atomic per warp.
    const int n = __popc(sel);
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int wbase = 0;
    if (lane == 31 && incl > 0) wbase = atomicAdd(n_out, incl);
    wbase = __shfl_sync(0xffffffffu, wbase, 31);
    int pos = wbase + incl - n;
#pragma unroll
    for (int i = 0; i < kTopkItems; ++i) {
      if (((sel >> i) & 1u) && pos < cap)
        out[pos] = (static_cast<unsigned long long>(key[i]) << 32) |
                   static_cast<uint32_t>(v0 + i);
      pos += (sel >> i) & 1u;
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ok_mine += __shfl_xor_sync(0xffffffffu, ok_mine, off);
  if (lane == 0 && ok_mine) atomicAdd(n_ok, ok_mine);
  __syncthreads();
}

// Candidate list of block (p, b): the allowed keys of its slice at or above a
// threshold (in no particular order), its count and the threshold.  A slice
// of more than two sample widths first tries a threshold read off a
// histogram of its first kTopkMinSlice tokens, with room for half as many
// again as the sample predicts; the extraction pass verifies it (at least
// min(K, allowed) keys pass, at most cap).  Otherwise, or when that check
// fails, exact radix histograms of the whole slice set the threshold.
__global__ void __launch_bounds__(kTopkThreads) topk_local_kernel(const TopkArgs a) {
  __shared__ TopkShared sh;
  __shared__ int n_out, n_ok;
  sm100::grid_dependency_wait();  // the logits
  const int p = blockIdx.x, b = blockIdx.y;
  const SampleLogitsParams &s = a.s;
  const uint32_t bg = static_cast<uint32_t>(s.b_off + b);
  const float *row = s.logits + static_cast<size_t>(b) * s.V;
  const int lo = p * a.slice, hi = imin(s.V, lo + a.slice);
  const bool vec = (s.V & 3) == 0;
  unsigned long long *out = a.cand + (static_cast<size_t>(b) * a.P + p) * a.cap;
  if (threadIdx.x == 0) {
    n_out = 0;
    n_ok = 0;
  }
  __syncthreads();

  uint32_t thr = 0u;
  bool done = false;
  const int len = hi - lo;
  if (len > 2 * kTopkMinSlice) {
    topk_slice_hist(s, row, bg, lo, lo + kTopkMinSlice, vec, 0u, 0u, 21, kTopkBins, sh);
    const long long want = static_cast<long long>(a.K) * kTopkMinSlice / len;
    const int target = static_cast<int>(want + want / 2 + 16);
    int above, count, ok_sample;
    const int d = topk_select_digit(kTopkBins, target, sh, &above, &count, &ok_sample);
    if (ok_sample > target) {
      const uint32_t lo_key = static_cast<uint32_t>(d) << 21;
      topk_extract(s, row, bg, lo, hi, vec, lo_key, false, 0, out, a.cap, &n_out, &n_ok, sh);
      const int got = n_out, allowed = n_ok;
      done = got >= imin(a.K, allowed) && got <= a.cap;
      if (done) {
        thr = got >= a.K ? lo_key : 0u;
      } else {
        __syncthreads();  // every thread has read the counts
        if (threadIdx.x == 0) {
          n_out = 0;
          n_ok = 0;
        }
        __syncthreads();
      }
    }
  }

  if (!done) {
    // Exact threshold: keys >= lo_key, or in exact mode keys > kb and the
    // first `take` keys equal to kb (lo_key = kb).
    uint32_t lo_key = 0u;
    bool exact = false;
    int take = 0;
    topk_slice_hist(s, row, bg, lo, hi, vec, 0u, 0u, 21, kTopkBins, sh);
    int above, count, allowed;
    const int d1 = topk_select_digit(kTopkBins, a.K, sh, &above, &count, &allowed);
    if (allowed > a.K) {
      uint32_t pre = static_cast<uint32_t>(d1) << 21;
      int k_rem = a.K - above;
      if (above + count <= a.cap) {
        lo_key = pre;
      } else {
        topk_slice_hist(s, row, bg, lo, hi, vec, pre, 0xFFE00000u, 10, kTopkBins, sh);
        int above2, count2, tot2;
        const int d2 = topk_select_digit(kTopkBins, k_rem, sh, &above2, &count2, &tot2);
        pre |= static_cast<uint32_t>(d2) << 10;
        above += above2;
        k_rem -= above2;
        if (above + count2 <= a.cap) {
          lo_key = pre;
        } else {
          topk_slice_hist(s, row, bg, lo, hi, vec, pre, 0xFFFFFC00u, 0, 1024, sh);
          int above3, count3, tot3;
          const int d3 = topk_select_digit(1024, k_rem, sh, &above3, &count3, &tot3);
          lo_key = pre | static_cast<uint32_t>(d3);
          exact = true;
          take = k_rem - above3;  // 1 <= take <= count3
        }
      }
      thr = lo_key;
    }
    topk_extract(s, row, bg, lo, hi, vec, lo_key, exact, take, out, a.cap, &n_out, &n_ok, sh);
  }
  if (threadIdx.x == 0) {
    const size_t at = static_cast<size_t>(b) * a.P + p;
    a.cnt[at] = imin(n_out, a.cap);
    a.thr[at] = thr;
  }
}

// A row's candidates for topk_row_kernel: kept in shared memory when they
// fit, else read from the blocks' lists (flat index i over the lists, whose
// offsets are in shared memory), keys below t0 excluded.
struct TopkRowCands {
  const unsigned long long *sm;     // kept entries, or nullptr
  const unsigned long long *lists;  // [P][cap]
  const int *offs;                  // P + 1 list offsets
  int P, cap;
  uint32_t t0;
  __device__ __forceinline__ bool entry(int i, unsigned long long &e) const {
    if (sm != nullptr) {
      e = sm[i];
      return true;
    }
    int q = 0, qe = P;  // the list holding flat index i: offs[q] <= i < offs[q + 1]
    while (qe - q > 1) {
      const int mid = (q + qe) >> 1;
      if (offs[mid] <= i) q = mid; else qe = mid;
    }
    e = __ldcg(lists + static_cast<size_t>(q) * cap + (i - offs[q]));
    return static_cast<uint32_t>(e >> 32) >= t0;
  }
};

// The k-th largest (1-based, k <= the participating count) of the 32-bit
// values of entries [0, n): MODE 0 the key of every entry; MODE 1 ~token of
// the entries whose key is kb (so the k-th largest is the k-th smallest
// token).  Three radix passes over bits 31-21, 20-10, 9-0; *n_above gets the
// count of larger values, *n_eq the count equal to the result.
template <int MODE>
__device__ uint32_t topk_row_kth(const TopkRowCands &c, int n, int k, uint32_t kb,
                                 TopkShared &sh, int *n_above, int *n_eq) {
  uint32_t pre = 0u, pmask = 0u;
  int above_total = 0, count = 0;
#pragma unroll 1
  for (int level = 0; level < 3; ++level) {
    const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
    const int nb = level == 2 ? 1024 : kTopkBins;
    for (int i = threadIdx.x; i < kTopkSubHists * nb; i += kTopkThreads) sh.hist[i] = 0;
    __syncthreads();
    int *my_hist = sh.hist + ((threadIdx.x >> 5) & (kTopkSubHists - 1)) * nb;
    for (int i = threadIdx.x; i < n; i += kTopkThreads) {
      unsigned long long e;
      if (!c.entry(i, e)) continue;
      const uint32_t key = static_cast<uint32_t>(e >> 32);
      if (MODE == 1 && key != kb) continue;
      const uint32_t v = MODE == 0 ? key : ~static_cast<uint32_t>(e);
      if ((v & pmask) == pre) atomicAdd(&my_hist[(v >> shift) & static_cast<uint32_t>(nb - 1)], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += kTopkThreads) {
      int t = 0;
#pragma unroll
      for (int h = 0; h < kTopkSubHists; ++h) t += sh.hist[h * nb + i];
      sh.hist[i] = t;
    }
    __syncthreads();
    int above, tot;
    const int d = topk_select_digit(nb, k, sh, &above, &count, &tot);
    pre |= static_cast<uint32_t>(d) << shift;
    pmask |= static_cast<uint32_t>(nb - 1) << shift;
    k -= above;
    above_total += above;
  }
  *n_above = above_total;
  *n_eq = count;
  return pre;
}

// Row b: keeps the candidates at or above the largest block threshold (the
// row's k-th largest key is at least every block's), selects the exact top
// K (ties toward the smaller token), draws their noise and writes the
// Gumbel-max token.
__global__ void __launch_bounds__(kTopkThreads) topk_row_kernel(const TopkArgs a) {
  __shared__ TopkShared sh;
  __shared__ int offs[kTopkMaxP + 1];
  __shared__ int n_kept, n_small;
  __shared__ unsigned int t0;
  __shared__ unsigned long long small[kTopkRowSmall];
  extern __shared__ unsigned long long kept[];  // kTopkRowCap entries
  // The kernel after this one may start launching now: a fused sampling
  // kernel launched as a programmatic dependent streams W meanwhile and
  // waits for this grid to complete before it loads H or touches the
  // workspace or the outputs this grid writes.
  sm100::launch_dependents();
  sm100::grid_dependency_wait();  // the candidate lists
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const SampleLogitsParams &s = a.s;
  const uint32_t bg = static_cast<uint32_t>(s.b_off + b);
  const unsigned long long *lists = a.cand + static_cast<size_t>(b) * a.P * a.cap;

  if (threadIdx.x == 0) {
    n_kept = 0;
    n_small = 0;
    t0 = 0u;
  }
  __syncthreads();
  int cq = 0;
  if (threadIdx.x < a.P) {
    cq = __ldcg(a.cnt + static_cast<size_t>(b) * a.P + threadIdx.x);
    atomicMax(&t0, __ldcg(a.thr + static_cast<size_t>(b) * a.P + threadIdx.x));
  }
  const int off = block_exclusive_scan(cq, sh.warp_sums, &sh.total);  // orders the writes above
  const int total = sh.total;
  if (threadIdx.x < a.P) offs[threadIdx.x] = off;
  if (threadIdx.x == 0) offs[a.P] = total;
  __syncthreads();

  // Keep the entries with key >= t0 in shared memory while they fit.
  TopkRowCands c{nullptr, lists, offs, a.P, a.cap, t0};
  for (int i0 = 0; i0 < total; i0 += kTopkThreads) {
    const int i = i0 + threadIdx.x;
    unsigned long long e = 0ull;
    const bool keep = i < total && c.entry(i, e);
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    int wbase = 0;
    if (lane == 0 && m) wbase = atomicAdd(&n_kept, __popc(m));
    wbase = __shfl_sync(0xffffffffu, wbase, 0);
    const int pos = wbase + __popc(m & ((1u << lane) - 1u));
    if (keep && pos < kTopkRowCap) kept[pos] = e;
  }
  __syncthreads();
  const int n_all = n_kept;
  int n = total;
  if (n_all <= kTopkRowCap) {
    c.sm = kept;
    n = n_all;
  }

  const bool all = n_all <= a.K;
  // One radix level over the kept keys (bits 31-21); when the keys at or
  // above the k-th largest key's digit are few, they are ranked directly:
  // rank = entries with a larger key, or the same key and a smaller token.
  bool by_rank = false;
  if (!all && c.sm != nullptr) {
    for (int i = threadIdx.x; i < kTopkSubHists * kTopkBins; i += kTopkThreads) sh.hist[i] = 0;
    __syncthreads();
    int *my_hist = sh.hist + ((threadIdx.x >> 5) & (kTopkSubHists - 1)) * kTopkBins;
    for (int i = threadIdx.x; i < n; i += kTopkThreads)
      atomicAdd(&my_hist[static_cast<uint32_t>(kept[i] >> 53)], 1);
    __syncthreads();
    for (int i = threadIdx.x; i < kTopkBins; i += kTopkThreads) {
      int t = 0;
#pragma unroll
      for (int h = 0; h < kTopkSubHists; ++h) t += sh.hist[h * kTopkBins + i];
      sh.hist[i] = t;
    }
    __syncthreads();
    int above, count, tot;
    const uint32_t d1 = static_cast<uint32_t>(topk_select_digit(kTopkBins, a.K, sh, &above, &count, &tot));
    if (above + count <= kTopkRowSmall) {
      by_rank = true;
      for (int i0 = 0; i0 < n; i0 += kTopkThreads) {
        const int i = i0 + threadIdx.x;
        const unsigned long long e = i < n ? kept[i] : 0ull;
        const bool keep = i < n && static_cast<uint32_t>(e >> 53) >= d1;
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        int wbase = 0;
        if (lane == 0 && m) wbase = atomicAdd(&n_small, __popc(m));
        wbase = __shfl_sync(0xffffffffu, wbase, 0);
        const int pos = wbase + __popc(m & ((1u << lane) - 1u));
        if (keep && pos < kTopkRowSmall) small[pos] = e;
      }
      __syncthreads();
      c.sm = small;
      n = n_small;  // == above + count
    }
  }
  uint32_t kb = 0u, ti = 0u;
  int take = 0, n_eq = 0;
  bool rank_ties = false;
  if (!all && !by_rank) {
    int n_above;
    kb = topk_row_kth<0>(c, n, a.K, 0u, sh, &n_above, &n_eq);
    take = a.K - n_above;  // 1 <= take <= n_eq
    if (take < n_eq) {
      rank_ties = true;
      int a2, e2;
      ti = topk_row_kth<1>(c, n, take, kb, sh, &a2, &e2);
    }
  }

  const uint64_t k64 =
      (s.row_seeds && FS_IN_BOUNDS(s.err, bg, s.rows_total)) ? s.row_seeds[bg] : s.seed;
  uint64_t best = 0ull;
  // Ranking: G consecutive lanes share an entry (G = 1024 / n rounded down to
  // a power of two, at most 32), each counting over every G-th entry.
  int gsh = 0;
  if (by_rank)
    while (gsh < 5 && (n << (gsh + 1)) <= kTopkThreads) ++gsh;
  const int G = 1 << gsh;
  const int per_pass = kTopkThreads >> gsh;
  for (int i0 = 0; i0 < n; i0 += per_pass) {  // block-uniform trip count
    const int i = i0 + (threadIdx.x >> gsh);
    const int sub = threadIdx.x & (G - 1);
    unsigned long long e = 0ull;
    const bool have = i < n && c.entry(i, e);
    const uint32_t key = static_cast<uint32_t>(e >> 32);
    bool sel;
    if (by_rank) {
      const uint32_t tok = static_cast<uint32_t>(e);
      int rank = 0;
      if (have) {
        for (int j = sub; j < n && rank < a.K; j += G) {
          const unsigned long long f = small[j];
          const uint32_t kf = static_cast<uint32_t>(f >> 32);
          rank += (kf > key || (kf == key && static_cast<uint32_t>(f) < tok)) ? 1 : 0;
        }
      }
      for (int o = G >> 1; o >= 1; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
      sel = have && sub == 0 && rank < a.K;
    } else {
      sel = have && (all || key > kb ||
                     (key == kb && (!rank_ties || ~static_cast<uint32_t>(e) >= ti)));
    }
    if (!sel) continue;
    const int v = static_cast<int>(static_cast<uint32_t>(e));
    const float l = __uint_as_float(order_bits_inv(key));
    const Philox4 ph = philox4x32_10(static_cast<uint32_t>(v) >> 2, bg, s.step, 0u,
                                     static_cast<uint32_t>(k64), static_cast<uint32_t>(k64 >> 32));
    const uint32_t w = (v & 3) == 0 ? ph.w0 : (v & 3) == 1 ? ph.w1 : (v & 3) == 2 ? ph.w2 : ph.w3;
    const float sc = fmaf(l, s.inv_temp, gumbel_from_u32(w));
    const uint64_t k = pack_key(__float_as_uint(sc), v);
    best = k > best ? k : best;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t x = __shfl_xor_sync(0xffffffffu, best, o);
    best = x > best ? x : best;
  }
  if (lane == 0) sh.warp_best[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t r = 0ull;
    for (int i = 0; i < kTopkThreads / 32; ++i) r = sh.warp_best[i] > r ? sh.warp_best[i] : r;
    s.out_idx[b] = key_token(r);
  }
}

cudaError_t launch_topk_sample(const SampleLogitsParams &s, int K, void *scratch,
                               cudaStream_t stream) {
  const TopkGeom g = topk_geom(s.B, s.V, K, s.num_sms);
  TopkArgs a;
  a.s = s;
  a.K = K;
  a.P = g.P;
  a.slice = g.slice;
  a.cap = g.cap;
  char *base = static_cast<char *>(scratch);
  const size_t lists = static_cast<size_t>(s.B) * g.P * g.cap * 8;
  a.cand = reinterpret_cast<unsigned long long *>(base);
  a.cnt = reinterpret_cast<int *>(base + lists);
  a.thr = reinterpret_cast<unsigned int *>(base + lists + static_cast<size_t>(s.B) * g.P * 4);
  const size_t row_smem = static_cast<size_t>(kTopkRowCap) * 8;  // above the default limit
  cudaError_t e = cudaFuncSetAttribute(topk_row_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(row_smem));
  if (e != cudaSuccess) return e;
  e = launch_dependent(topk_local_kernel, dim3(g.P, s.B), dim3(kTopkThreads), stream, a);
  if (e != cudaSuccess) return e;
  return launch_dependent_smem(topk_row_kernel, dim3(s.B), dim3(kTopkThreads), row_smem, stream,
                               a);
}
// ---------------------------------------------------------------------------
// Two-kernel reduction (an A/B alternative to the last CTA's ticket): one
// thread per (row, sample) reads the published maximum and re-zeroes it.
// ---------------------------------------------------------------------------
__global__ void decode_published_kernel(unsigned long long *keys, int B, int S, int32_t *out_idx,
                                        long long *out_keys, int *err, int keys_cap) {
  sm100::launch_dependents();
  sm100::grid_dependency_wait();  // the fused kernel's published keys
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * S) return;
  const int b = i / S;
  const int smp = i - b * S;
  if (!FS_IN_BOUNDS(err, smp * kMaxBN + b, keys_cap)) return;
  const unsigned long long kb = atomicExch(keys + smp * kMaxBN + b, 0ull);
  if (out_keys != nullptr)
    out_keys[i] = static_cast<long long>(kb ^ 0x8000000000000000ull);  // signed order
  else
    out_idx[i] = key_token(kb);
}

cudaError_t launch_decode_published(unsigned long long *keys, int B, int num_samples,
                                    int32_t *out_idx, long long *out_keys, int *err,
                                    int keys_cap, cudaStream_t stream) {
  const int n = B * num_samples;
  return launch_dependent(decode_published_kernel, dim3((n + 255) / 256), dim3(256), stream, keys,
                          B, num_samples, out_idx, out_keys, err, keys_cap);
}

// ---------------------------------------------------------------------------
// Vocabulary shards: tokens from the reduced keys.
// ---------------------------------------------------------------------------
__global__ void keys_to_tokens_kernel(const long long *keys, int B, int32_t *out_idx) {
  // The kernel after this one may start launching now: a fused sampling
  // kernel launched as a programmatic dependent streams W meanwhile and
  // waits for this grid to complete before it loads H or touches the
  // workspace or the outputs this grid writes.
  sm100::launch_dependents();
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
// Tensor-parallel exchange: this rank's wait for a call's tokens.
// ---------------------------------------------------------------------------
// Acquire load at system scope (a word another GPU stores with release
// semantics after the data it guards), a relaxed load of a guarded word, and
// the GPU's global nanosecond timer.
__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t *addr) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}

__device__ __forceinline__ int32_t ld_relaxed_sys(const int32_t *addr) {
  int32_t v;
  asm volatile("ld.relaxed.sys.global.b32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long global_time_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// One block, launched after this rank's sampling kernel.  Thread 0 polls the
// area's flag -- stored with release semantics at system scope, after the
// tokens, by whichever rank's last CTA completed the area -- until it reaches
// seq + 1 (compared modulo 2^32) or the time limit passes; every poll sleeps
// a little, and the number of polls is capped as well.  Then the block copies
// the tokens of the call's half of the area, or, if the limit passed, writes
// -1 for every row and marks the call failed in the area.
__global__ void __launch_bounds__(256) tp_wait_kernel(TpArea *area, int B, uint32_t seq,
                                                      int32_t *out_idx,
                                                      unsigned long long limit_ns,
                                                      unsigned long long max_polls) {
  __shared__ int late;
  const uint32_t want = seq + 1u;
  if (threadIdx.x == 0) {
    const unsigned long long t0 = global_time_ns();
    int timed_out = 0;
    unsigned nap = 32;
    for (unsigned long long n = 0;; ++n) {
      if (static_cast<int32_t>(ld_acquire_sys(&area->flag) - want) >= 0) break;
      if (n >= max_polls || global_time_ns() - t0 >= limit_ns) {
        timed_out = 1;
        break;
      }
      __nanosleep(nap);
      if (nap < 1024) nap *= 2;
    }
    late = timed_out;
  }
  __syncthreads();
  const int half = static_cast<int>(seq & 1u);
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    if (late) {
      out_idx[b] = -1;
    } else {
      (void)ld_acquire_sys(&area->flag);  // orders this thread's token load after the flag
      out_idx[b] = ld_relaxed_sys(&area->tokens[half][b]);
    }
  }
  if (late && threadIdx.x == 0) atomicExch(&area->failed, want);
}

cudaError_t launch_tp_wait(TpArea *area, int B, uint32_t seq, int32_t *out_idx,
                           uint32_t timeout_us, cudaStream_t stream) {
  const unsigned long long limit_ns = 1000ull * timeout_us;
  const unsigned long long max_polls = 64ull * timeout_us + 4096ull;
  tp_wait_kernel<<<1, 256, 0, stream>>>(area, B, seq, out_idx, limit_ns, max_polls);
  return cudaGetLastError();
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
