// api.cu -- the C ABI of libfmms (declared in include/fmms.h): argument
// validation, workspace management, TMA tensor maps and kernel dispatch.
// Nothing here computes a sampling step; every step runs in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "fmms.h"
#include "fmms_common.cuh"
#include "launch.h"

namespace {

using fmms::FmmsParams;
using fmms::Schedule;

// ------------------------------------------------------------- device state
struct DeviceState {
  bool init = false;
  int sms = 0;
  int cc_major = 0;
  void *ws = nullptr;       // library-owned workspace
  size_t ws_bytes = 0;
  void *h_stage[2] = {nullptr, nullptr};  // fs_sample_host: device copies of H, by call parity
  size_t h_stage_bytes[2] = {0, 0};
  void *o_stage = nullptr;  // fs_sample_host: device tokens
  size_t o_stage_bytes = 0;
  void *topk_scratch = nullptr;  // fs_sample_topk: per-block candidate lists and counts
  void *forced_logits = nullptr;  // FS_FORCE_PATH=unfused: fp32 logits of flat calls
  size_t forced_logits_bytes = 0;
  size_t topk_scratch_bytes = 0;
  // fs_sample_host: H is copied on copy_stream while the kernel already
  // streams W; h_flags[k] takes the call's epoch once the copy into
  // h_stage[k] has landed.  Calls alternate between the two buffers, and
  // kernel_done[k] keeps a copy off h_stage[k] until the kernel that last
  // read it (two calls back) has finished, so a call's copy runs during the
  // previous call's kernel.
  bool host_overlap_init = false;
  bool host_overlap = false;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t kernel_done[2] = {nullptr, nullptr};
  uint32_t *h_flags = nullptr;  // device words [2]: epoch of the H copy that has landed
  uint32_t h_epoch = 0;
  uint32_t h_calls = 0;
  int pair_units[2][fmms::kMaxBN / 16];  // resident CTA pairs [flat, grouped][tile / 16 - 1]; -1: unknown
  DeviceState() {
    for (auto &row : pair_units)
      for (int &u : row) u = -1;
  }
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
// The device attributes are read once per device, also when the first calls
// come from several threads at once (not every entry point holds g_mu).
std::once_flag g_dev_once[kMaxDevices];

fs_status get_device(DeviceState **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FS_ERR_CUDA;
  DeviceState &st = g_dev[dev];
  std::call_once(g_dev_once[dev], [&st, dev] {
    st.init = cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
              cudaDeviceGetAttribute(&st.cc_major, cudaDevAttrComputeCapabilityMajor, dev) ==
                  cudaSuccess;
  });
  if (!st.init) return FS_ERR_CUDA;
  if (st.cc_major != 10) return FS_ERR_UNSUPPORTED;  // built for sm_100a only
  *out = &st;
  return FS_OK;
}

// Host-side fault injection for failure-detection tests.  FS_FAULT=alloc
// makes every device allocation the library would make fail, FS_FAULT=launch
// every call that would enqueue work; such a call returns FS_ERR_CUDA before
// it touches the GPU.  The environment is read once; fs_test_inject_fault
// overrides it.
constexpr int kFaultNone = 0, kFaultAlloc = 1, kFaultLaunch = 2;
std::atomic<int> g_fault{-1};  // -1: environment not read yet

int fault_mode() {
  int f = g_fault.load(std::memory_order_relaxed);
  if (f >= 0) return f;
  const char *e = getenv("FS_FAULT");
  f = kFaultNone;
  if (e != nullptr && strcmp(e, "alloc") == 0) f = kFaultAlloc;
  if (e != nullptr && strcmp(e, "launch") == 0) f = kFaultLaunch;
  int expect = -1;
  g_fault.compare_exchange_strong(expect, f);
  return g_fault.load(std::memory_order_relaxed);
}

bool launch_fault() { return fault_mode() == kFaultLaunch; }

// Grows a library-owned device buffer; new memory is zero-filled.
fs_status grow(void **buf, size_t *have, size_t need) {
  if (*have >= need) return FS_OK;
  if (fault_mode() == kFaultAlloc) return FS_ERR_CUDA;
  if (*buf) {
    cudaDeviceSynchronize();
    cudaFree(*buf);
    *buf = nullptr;
    *have = 0;
  }
  if (cudaMalloc(buf, need) != cudaSuccess) return FS_ERR_CUDA;
  if (cudaMemset(*buf, 0, need) != cudaSuccess) return FS_ERR_CUDA;
  *have = need;
  return FS_OK;
}

// ----------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuStreamWriteValue32: a 32-bit store done by the copy engine in stream
// order, so it needs no SM while the persistent kernel holds all of them.
using StreamWriteValue32Fn = CUresult (*)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);

StreamWriteValue32Fn write_value_fn() {
  static StreamWriteValue32Fn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuStreamWriteValue32", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<StreamWriteValue32Fn>(p);
  });
  return fn;
}

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A bf16 matrix [rows][inner] read in boxes of [box_rows][64] with the
// 128-byte swizzle; out-of-range elements read as zero.
struct TmapKey {
  const void *ptr;
  uint64_t inner, rows;
  uint32_t box_rows;
  int dev;
};

struct TmapEntry {
  TmapKey key;
  CUtensorMap map;
  bool used = false;
};

constexpr int kTmapCache = 64;
TmapEntry g_tmaps[kTmapCache];
int g_tmap_next = 0;

fs_status tensor_map(CUtensorMap *out, const void *ptr, uint64_t inner, uint64_t rows,
                     uint32_t box_rows) {
  int dev = 0;
  cudaGetDevice(&dev);
  for (auto &e : g_tmaps) {
    if (e.used && e.key.ptr == ptr && e.key.inner == inner && e.key.rows == rows &&
        e.key.box_rows == box_rows && e.key.dev == dev) {
      *out = e.map;
      return FS_OK;
    }
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FS_ERR_CUDA;
  CUtensorMap m;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(fmms::kBlockK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return FS_ERR_CUDA;
  TmapEntry &e = g_tmaps[g_tmap_next];
  g_tmap_next = (g_tmap_next + 1) % kTmapCache;
  e.key = TmapKey{ptr, inner, rows, box_rows, dev};
  e.map = m;
  e.used = true;
  *out = m;
  return FS_OK;
}

// ------------------------------------------------------------ validation
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fs_status validate(const void *H, const void *W, int B, int d, int V, float T, const void *out) {
  if (!H || !W || !out) return FS_ERR_INVALID_ARG;
  if (B < 1 || V < 1 || d < 8 || (d % 8) != 0) return FS_ERR_INVALID_ARG;
  if (!(T > 0.f) || !isfinite(T)) return FS_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(W)) return FS_ERR_INVALID_ARG;
  return FS_OK;
}

struct Workspace {
  int *err;
  unsigned int *ticket;
  unsigned long long *keys;
  fmms::GroupPartial *partials;
  unsigned long long *gkeys;
};

Workspace carve(void *ws, int B, int G, int num_ctas, int samples, bool grouped) {
  char *b = static_cast<char *>(ws);
  (void)samples;
  const size_t keys_bytes = static_cast<size_t>(fmms::kWsKeysRegion);  // fixed layout
  Workspace w;
  w.err = reinterpret_cast<int *>(b);
  w.ticket = reinterpret_cast<unsigned int *>(b + 4);
  w.keys = reinterpret_cast<unsigned long long *>(b + fmms::kWsHeader);
  w.partials = reinterpret_cast<fmms::GroupPartial *>(b + fmms::kWsHeader + keys_bytes);
  w.gkeys = (grouped && fmms::ws_gkeys_bytes(B, G) > 0)
                ? reinterpret_cast<unsigned long long *>(
                      b + fmms::kWsHeader + keys_bytes + fmms::ws_partials_bytes(B, G, num_ctas))
                : nullptr;
  return w;
}

fs_status resolve_workspace(DeviceState *st, const Schedule &sch, int B, int samples,
                            bool grouped, void *ws, size_t ws_bytes, void **out) {
  const size_t need =
      static_cast<size_t>(fmms::workspace_bytes_for(B, sch.G, sch.num_ctas, samples, grouped));
  if (ws == nullptr) {
    fs_status s = grow(&st->ws, &st->ws_bytes, need);
    if (s != FS_OK) return s;
    *out = st->ws;
    return FS_OK;
  }
  if (ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FS_ERR_WORKSPACE;
  *out = ws;
  return FS_OK;
}

// Set for the duration of fs_test_stalled_sample, or between
// fs_test_stall_loads(1) and fs_test_stall_loads(0) (under g_mu).
bool g_test_no_loads = false;
bool g_test_stall = false;

// fs_set_cta_pairs: -1 automatic, 0 never, 1 whenever the call allows it.
int g_pair_policy = -1;
// fs_set_programmatic_launch: 1 (default) launch the fused kernel as a
// programmatic dependent of the kernel ahead of it in the stream (launches
// with batch tiles of up to 128 rows), 0 plain stream order.
int g_pdl_policy = 1;
// fs_set_partial_merge: -1 automatic, 0 never, 1 always (single CTAs, <= 64 rows).
int g_merge_policy = -1;

// FS_FORCE_PATH (environment, read once at the first sampling call): a
// comma-separated list that sets the initial execution-path choices for A/B
// runs without code changes -- "unfused" (flat single-sample calls fs_sample
// and fs_sample_ex run the two-kernel measurement mode: fp32 logits through
// HBM, then the sampling kernel) or "fused"; "pairs" or "single" (as
// fs_set_cta_pairs(1 / 0)); "merge" or "nomerge" (fs_set_partial_merge);
// "plain" or "programmatic" (fs_set_programmatic_launch); "twokernel" or
// "lastcta" (flat calls reduce the per-row maxima in a second kernel, or in
// the fused kernel's last CTA).  Unknown words are ignored.  The fs_set_*
// calls still override it afterwards.
bool g_force_unfused = false;
bool g_two_kernel_reduce = false;
std::once_flag g_force_once;

void read_force_path() {
  std::call_once(g_force_once, [] {
    const char *e = getenv("FS_FORCE_PATH");
    if (e == nullptr) return;
    const char *p = e;
    while (*p) {
      const char *q = p;
      while (*q && *q != ',') ++q;
      const size_t n = static_cast<size_t>(q - p);
      auto is = [&](const char *w) { return strlen(w) == n && strncmp(p, w, n) == 0; };
      if (is("unfused")) g_force_unfused = true;
      if (is("fused")) g_force_unfused = false;
      if (is("pairs")) g_pair_policy = 1;
      if (is("single")) g_pair_policy = 0;
      if (is("merge")) g_merge_policy = 1;
      if (is("nomerge")) g_merge_policy = 0;
      if (is("twokernel")) g_two_kernel_reduce = true;
      if (is("lastcta")) g_two_kernel_reduce = false;
      if (is("plain")) g_pdl_policy = 0;
      if (is("programmatic")) g_pdl_policy = 1;
      p = *q ? q + 1 : q;
    }
  });
}

int bn_index(int BN) { return BN / 16 - 1; }

// CTA pairs of the BN pair kernel of `mode` that fit on the device at once
// (0: none).
int pair_units(DeviceState *st, int mode, int BN) {
  int &u = st->pair_units[mode == fmms::kModeGrouped ? 1 : 0][bn_index(BN)];
  if (u < 0) {
    int n = 0;
    if (fmms::fmms_pair_units(mode, BN, &n) != cudaSuccess) {
      cudaGetLastError();  // clear the error; the single-CTA kernel is used
      n = 0;
    }
    u = fmms::imin(n, st->sms / 2);
  }
  return u;
}

// Flat and grouped calls with a batch tile of 112 or more rows run on CTA
// pairs: each SM then stages half of H per stage, which halves the batch
// operand's L2 traffic and the MMA issues per byte of W where the tensor
// cores are busy.  Measured (200 back-to-back calls, single CTAs / pairs):
// Qwen3-8B head B=96 208.8 / 212.4 us, B=112 239.3 / 218.6 us, B=128
// 248.9 / 226.9 us; Qwen3-1.7B head B=96 110.7 / 110.5, B=112 126.9 / 113.6.
bool use_pairs(int mode, int BN) {
  if (mode == fmms::kModeLogits || g_pair_policy == 0) return false;
  return g_pair_policy == 1 || BN >= 112;
}

// Options of vocabulary-shard and multi-sample calls.
struct ShardOpts {
  int vocab_offset = 0;         // global token index of W row 0
  int V_total = 0;              // full vocabulary (0: V); sets the mask row length
  long long *out_keys = nullptr;  // write packed keys instead of tokens
  int num_samples = 1;          // samples per row (flat mode)
  int top_k = 0;                // logits mode: top-k selection instead of full sampling
  const uint32_t *h_ready = nullptr;  // H arriving in chunks (fs_sample_host), else null
  uint32_t h_epoch = 0;
  int h_chunk_subs = 0;
  int tp_world = 0;             // fused vocabulary-parallel exchange (flat mode)
  uint32_t tp_seq = 0;
  void *const *tp_areas = nullptr;
};

// Whether the kernel variant with merged 8-row partial tiles pays for this
// vocabulary split: at least one CTA in ten starts a segment with an 8-row
// partial tile (the Qwen3 heads: 48 of 148).  Elsewhere its extra slot per
// stage only costs ring space.  merge_partials applies the policy switch and
// remembers the last few answers.
bool merge_rule(const Schedule &sch) {
  int with = 0;
  for (int c = 0; c < sch.num_ctas; ++c) {
    fmms::TileIter it(sch, c, 1);
    fmms::Tile t;
    while (it.next(t)) {
      if (t.pstart >= 0) {
        ++with;
        break;
      }
    }
  }
  return with * 10 >= sch.num_ctas;
}

bool merge_partials(const Schedule &sch) {
  if (g_merge_policy >= 0) return g_merge_policy == 1;
  struct Entry {
    int V, G, num_ctas;
    bool merge;
  };
  static Entry memo[8];
  static int memo_next = 0, memo_used = 0;
  for (int i = 0; i < memo_used; ++i)
    if (memo[i].V == sch.V && memo[i].G == sch.G && memo[i].num_ctas == sch.num_ctas)
      return memo[i].merge;
  const bool merge = merge_rule(sch);
  memo[memo_next] = Entry{sch.V, sch.G, sch.num_ctas, merge};
  memo_next = (memo_next + 1) % 8;
  if (memo_used < 8) ++memo_used;
  return merge;
}

// The fused path in all three modes, chunked over 256 batch rows.
fs_status run_locked(int mode, const void *H, const void *W, int B, int d, int V, int G,
                     float T, uint64_t seed, const uint64_t *row_seeds, uint32_t step,
                     const uint32_t *mask, int32_t *out_idx, fs_group_summary *summary,
                     float *logits, void *ws, size_t ws_bytes, cudaStream_t stream,
                     const ShardOpts &shard = ShardOpts());

fs_status run(int mode, const void *H, const void *W, int B, int d, int V, int G, float T,
              uint64_t seed, const uint64_t *row_seeds, uint32_t step, const uint32_t *mask,
              int32_t *out_idx, fs_group_summary *summary, float *logits, void *ws,
              size_t ws_bytes, cudaStream_t stream) {
  read_force_path();
  std::lock_guard<std::mutex> lock(g_mu);
  return run_locked(mode, H, W, B, d, V, G, T, seed, row_seeds, step, mask, out_idx, summary,
                    logits, ws, ws_bytes, stream);
}

fs_status run_locked(int mode, const void *H, const void *W, int B, int d, int V, int G,
                     float T, uint64_t seed, const uint64_t *row_seeds, uint32_t step,
                     const uint32_t *mask, int32_t *out_idx, fs_group_summary *summary,
                     float *logits, void *ws, size_t ws_bytes, cudaStream_t stream,
                     const ShardOpts &shard) {
  if (launch_fault()) return FS_ERR_CUDA;
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  const Schedule sch = fmms::make_schedule(V, mode == fmms::kModeGrouped ? G : 1, st->sms);
  void *wsp = nullptr;
  const int S = shard.num_samples;
  const bool grouped = mode == fmms::kModeGrouped;
  s = resolve_workspace(st, sch, B, S, grouped, ws, ws_bytes, &wsp);
  if (s != FS_OK) return s;
  const Workspace w = carve(wsp, B, sch.G, sch.num_ctas, S, grouped);

  CUtensorMap tw;
  fmms::PartMaps twp;
  if ((s = tensor_map(&tw, W, d, V, fmms::kTileM)) != FS_OK) return s;
  for (int b = 0; b < 4; ++b)
    if ((s = tensor_map(&twp.box[b], W, d, V, fmms::kGranule << b)) != FS_OK) return s;

  for (int b0 = 0; b0 < B; b0 += fmms::kMaxBN) {
    const int Bc = fmms::imin(fmms::kMaxBN, B - b0);
    const int BN = fmms::fmms_batch_tile(Bc);
    const int units = use_pairs(mode, BN) ? pair_units(st, mode, BN) : 0;
    const bool pair = units > 0;
    CUtensorMap th;
    if ((s = tensor_map(&th, H, d, B, pair ? BN / 2 : BN)) != FS_OK) return s;
    FmmsParams p;
    memset(&p, 0, sizeof p);
    p.B = Bc;
    p.b_off = b0;
    p.d = d;
    p.V = V;
    p.G = sch.G;
    p.num_ctas = sch.num_ctas;
    p.ngran = sch.ngran;
    p.nk = (d + fmms::kBlockK - 1) / fmms::kBlockK;
    p.inv_temp = 1.0f / T;
    p.step = step;
    p.seed = seed;
    p.row_seeds = row_seeds;
    p.mask = mask;
    p.mask_words = ((shard.V_total > 0 ? shard.V_total : V) + 31) / 32;
    p.out_idx = out_idx ? out_idx + static_cast<size_t>(b0) * S : nullptr;
    p.keys = w.keys;
    p.ticket = w.ticket;
    p.err = w.err;
    p.partials = w.partials;
    p.gkeys = mode == fmms::kModeGrouped ? w.gkeys : nullptr;
    p.logits = logits ? logits + static_cast<size_t>(b0) * V : nullptr;
    p.test_no_loads = (g_test_no_loads || g_test_stall) ? 1 : 0;
    // Programmatic launch where the kernel streams W at the bandwidth limit
    // (batch tiles up to 128 rows: Qwen3-8B head B=1 183.6 -> 179.8 us,
    // B=64 192.1 -> 188.8 us, Qwen3-1.7B head B=64 103.2 -> 99.5 us, tiny
    // head 13-16 -> 12.4 us); at 256 rows, tensor-bound, the overlap
    // measured 2-3 % slower.
    p.pdl = (g_pdl_policy != 0 && BN <= 128) ? 1 : 0;
    // The two-kernel reduction applies to flat launches that end in tokens
    // or keys of this device (not the fused exchange).
    const bool two_kernel = g_two_kernel_reduce && mode == fmms::kModeFlat && shard.tp_world == 0;
    p.no_ticket = two_kernel ? 1 : 0;
    p.vocab_offset = shard.vocab_offset;
    p.out_keys = shard.out_keys ? shard.out_keys + static_cast<size_t>(b0) * S : nullptr;
    p.num_samples = S;
    p.h_ready = shard.h_ready;
    p.h_epoch = shard.h_epoch;
    p.h_chunk_subs = shard.h_chunk_subs;
    p.tp_world = shard.tp_world;
    p.tp_seq = shard.tp_seq;
    for (int r = 0; r < shard.tp_world; ++r)
      p.tp_area[r] = static_cast<fmms::TpArea *>(shard.tp_areas[r]);
    {
      const long long rows = fmms::imin(B, fmms::kMaxBN);
      p.rows_total = B;
      p.keys_cap = grouped ? fmms::kWsKeysRegion / 8 : S * fmms::kMaxBN;
      p.partials_cap = fmms::ws_partials_bytes(B, sch.G, sch.num_ctas) /
                       static_cast<long long>(sizeof(fmms::GroupPartial));
      p.gkeys_cap = fmms::ws_gkeys_bytes(B, sch.G) / 8;
      p.out_cap = Bc * S;
      p.logits_cap = static_cast<long long>(Bc) * V;
      (void)rows;
    }
    const int pair_units_used = pair ? fmms::make_schedule(V, sch.G, units).num_ctas : 0;
    if (pair) {
      p.num_ctas = 2 * pair_units_used;
      if (fmms::launch_fmms_pair(mode, BN, tw, twp, th, p, stream) != cudaSuccess)
        return FS_ERR_CUDA;
    } else {
      if (fmms::launch_fmms(mode, BN, merge_partials(sch), tw, twp, th, p, stream) != cudaSuccess)
        return FS_ERR_CUDA;
    }

    if (two_kernel) {
      if (fmms::launch_decode_published(w.keys, Bc, S, p.out_idx, p.out_keys, w.err, p.keys_cap,
                                        stream) != cudaSuccess)
        return FS_ERR_CUDA;
    } else if (mode == fmms::kModeGrouped) {
      fmms::MergeParams m;
      m.partials = w.partials;
      m.gkeys = w.gkeys;
      m.B = Bc;
      m.b_off = b0;
      m.V = V;
      m.G = sch.G;
      m.num_ctas = pair ? pair_units_used : sch.num_ctas;
      m.pair = pair ? 1 : 0;
      m.ngran = sch.ngran;
      m.seed = seed;
      m.row_seeds = row_seeds;
      m.step = step;
      m.out_idx = out_idx ? out_idx + b0 : nullptr;
      m.summary = summary ? static_cast<void *>(summary + static_cast<size_t>(b0) * sch.G) : nullptr;
      m.err = w.err;
      m.partials_cap = p.partials_cap;
      m.gkeys_cap = p.gkeys_cap;
      m.rows_total = B;
      if (fmms::launch_group_merge(m, stream) != cudaSuccess) return FS_ERR_CUDA;
    } else if (mode == fmms::kModeLogits) {
      fmms::SampleLogitsParams sp;
      sp.logits = p.logits;
      sp.B = Bc;
      sp.b_off = b0;
      sp.V = V;
      sp.inv_temp = p.inv_temp;
      sp.seed = seed;
      sp.row_seeds = row_seeds;
      sp.step = step;
      sp.mask = mask;
      sp.mask_words = p.mask_words;
      sp.keys = w.keys;
      sp.ticket = w.ticket;
      sp.out_idx = out_idx + b0;
      sp.num_sms = st->sms;
      sp.err = w.err;
      sp.rows_total = B;
      cudaError_t e;
      if (shard.top_k > 0) {
        s = grow(&st->topk_scratch, &st->topk_scratch_bytes,
                 fmms::topk_scratch_bytes(Bc, V, shard.top_k, st->sms));
        if (s != FS_OK) return s;
        e = fmms::launch_topk_sample(sp, shard.top_k, st->topk_scratch, stream);
      } else {
        e = fmms::launch_sample_logits(sp, stream);
      }
      if (e != cudaSuccess) return FS_ERR_CUDA;
    }
  }
  return FS_OK;
}

}  // namespace

extern "C" {

namespace {
// A flat single-sample call: the fused kernel, or with FS_FORCE_PATH=unfused
// the two-kernel mode with a library-owned logits buffer (same tokens).
fs_status run_flat(const void *H, const void *W, int B, int d, int V, float T, uint64_t seed,
                   const uint64_t *row_seeds, uint32_t step, const uint32_t *mask,
                   int32_t *out_idx, void *ws, size_t ws_bytes, cudaStream_t stream) {
  read_force_path();
  if (!g_force_unfused)
    return run(fmms::kModeFlat, H, W, B, d, V, 1, T, seed, row_seeds, step, mask, out_idx,
               nullptr, nullptr, ws, ws_bytes, stream);
  if (launch_fault()) return FS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  const size_t bytes = static_cast<size_t>(B) * V * sizeof(float);
  if ((s = grow(&st->forced_logits, &st->forced_logits_bytes, bytes)) != FS_OK) return s;
  ShardOpts o;
  s = run_locked(fmms::kModeLogits, H, W, B, d, V, 1, T, seed, row_seeds, step, mask, out_idx,
                 nullptr, static_cast<float *>(st->forced_logits), ws, ws_bytes, stream, o);
  if (s != FS_OK) return s;
  return FS_OK;
}
}  // namespace

fs_status fs_sample(const void *H, const void *W, int B, int d, int V, float temperature,
                    uint64_t seed, uint32_t step, const uint32_t *mask_bits, int32_t *out_idx,
                    fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, temperature, out_idx);
  if (s != FS_OK) return s;
  return run_flat(H, W, B, d, V, temperature, seed, nullptr, step, mask_bits, out_idx, nullptr,
                  0, static_cast<cudaStream_t>(stream));
}

fs_status fs_sample_ex(const void *H, const void *W, int B, int d, int V, float temperature,
                       uint64_t seed, const uint64_t *row_seeds, uint32_t step,
                       const uint32_t *mask_bits, int32_t *out_idx, void *workspace,
                       size_t workspace_bytes, fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, temperature, out_idx);
  if (s != FS_OK) return s;
  return run_flat(H, W, B, d, V, temperature, seed, row_seeds, step, mask_bits, out_idx,
                  workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

fs_status fs_sample_grouped(const void *H, const void *W, int B, int d, int V, int G,
                            float temperature, uint64_t seed, const uint64_t *row_seeds,
                            uint32_t step, const uint32_t *mask_bits, int32_t *out_idx,
                            fs_group_summary *out_summary, void *workspace, size_t workspace_bytes,
                            fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, temperature, out_idx);
  if (s != FS_OK) return s;
  if (G < 1 || G > V) return FS_ERR_INVALID_ARG;
  return run(fmms::kModeGrouped, H, W, B, d, V, G, temperature, seed, row_seeds, step, mask_bits,
             out_idx, out_summary, nullptr, workspace, workspace_bytes,
             static_cast<cudaStream_t>(stream));
}

fs_status fs_sample_unfused(const void *H, const void *W, int B, int d, int V, float temperature,
                            uint64_t seed, const uint64_t *row_seeds, uint32_t step,
                            const uint32_t *mask_bits, int32_t *out_idx, float *logits,
                            void *workspace, size_t workspace_bytes, fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, temperature, out_idx);
  if (s != FS_OK) return s;
  if (!logits) return FS_ERR_INVALID_ARG;
  return run(fmms::kModeLogits, H, W, B, d, V, 1, temperature, seed, row_seeds, step, mask_bits,
             out_idx, nullptr, logits, workspace, workspace_bytes,
             static_cast<cudaStream_t>(stream));
}

fs_status fs_sample_host(const void *H_host, const void *W, int B, int d, int V,
                         float temperature, uint64_t seed, const uint64_t *row_seeds,
                         uint32_t step, const uint32_t *mask_bits, int32_t *out_idx_host,
                         fs_stream_t stream) {
  if (!H_host || !out_idx_host) return FS_ERR_INVALID_ARG;
  if (B < 1 || V < 1 || d < 8 || (d % 8) != 0) return FS_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !isfinite(temperature) || !W || !aligned16(W))
    return FS_ERR_INVALID_ARG;
  if (launch_fault()) return FS_ERR_CUDA;
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  const size_t hbytes = static_cast<size_t>(B) * d * 2;
  const int hb = static_cast<int>(st->h_calls++ & 1u);
  if ((s = grow(&st->h_stage[hb], &st->h_stage_bytes[hb], hbytes)) != FS_OK) return s;
  if ((s = grow(&st->o_stage, &st->o_stage_bytes, static_cast<size_t>(B) * 4)) != FS_OK) return s;
  char *hdev = static_cast<char *>(st->h_stage[hb]);
  int32_t *odev = static_cast<int32_t *>(st->o_stage);

  if (!st->host_overlap_init) {
    st->host_overlap_init = true;
    st->host_overlap =
        write_value_fn() != nullptr &&
        cudaStreamCreateWithFlags(&st->copy_stream, cudaStreamNonBlocking) == cudaSuccess &&
        cudaEventCreateWithFlags(&st->kernel_done[0], cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&st->kernel_done[1], cudaEventDisableTiming) == cudaSuccess &&
        cudaMalloc(&st->h_flags, 2 * sizeof(uint32_t)) == cudaSuccess &&
        cudaMemset(st->h_flags, 0, 2 * sizeof(uint32_t)) == cudaSuccess &&
        cudaDeviceSynchronize() == cudaSuccess;
  }

  ShardOpts opts;
  if (st->host_overlap) {
    // H is copied on the library's copy stream into this call's staging
    // buffer once the kernel two calls back is done with it, and a
    // copy-engine write then sets the buffer's flag to this call's epoch.
    // The kernel, launched at once, streams W from its start and loads H
    // once the flag holds the epoch, so the copy overlaps the previous
    // call's kernel and this one's first W loads.  (Copying H in
    // several K-column chunks, each with its own flag, measured slower: 2-D
    // copies of 64-row strips and the extra waits cost more than they hid.)
    const int nk = (d + fmms::kBlockK - 1) / fmms::kBlockK;
    const uint32_t epoch = ++st->h_epoch == 0 ? ++st->h_epoch : st->h_epoch;
    if (cudaStreamWaitEvent(st->copy_stream, st->kernel_done[hb], 0) != cudaSuccess)
      return FS_ERR_CUDA;
    if (cudaMemcpyAsync(hdev, H_host, hbytes, cudaMemcpyHostToDevice, st->copy_stream) !=
        cudaSuccess)
      return FS_ERR_CUDA;
    if (write_value_fn()(reinterpret_cast<CUstream>(st->copy_stream),
                         reinterpret_cast<CUdeviceptr>(st->h_flags + hb), epoch, 0) !=
        CUDA_SUCCESS)
      return FS_ERR_CUDA;
    opts.h_ready = st->h_flags + hb;
    opts.h_epoch = epoch;
    opts.h_chunk_subs = nk;
  } else {
    if (cudaMemcpyAsync(hdev, H_host, hbytes, cudaMemcpyHostToDevice, st_) != cudaSuccess)
      return FS_ERR_CUDA;
  }
  // Page-locked token buffer: the kernel's last CTA stores the tokens into it
  // directly over PCIe (no separate device-to-host copy); otherwise they go
  // through the device staging buffer and a copy.
  cudaPointerAttributes pa;
  const bool direct = cudaPointerGetAttributes(&pa, out_idx_host) == cudaSuccess &&
                      pa.type == cudaMemoryTypeHost && pa.devicePointer != nullptr;
  if (!direct) cudaGetLastError();  // clear a lookup error on pageable memory
  int32_t *out_dev = direct ? static_cast<int32_t *>(pa.devicePointer) : odev;
  s = run_locked(fmms::kModeFlat, hdev, W, B, d, V, 1, temperature, seed, row_seeds, step,
                 mask_bits, out_dev, nullptr, nullptr, nullptr, 0, st_, opts);
  if (s != FS_OK) return s;
  if (st->host_overlap && cudaEventRecord(st->kernel_done[hb], st_) != cudaSuccess)
    return FS_ERR_CUDA;
  if (!direct && cudaMemcpyAsync(out_idx_host, odev, static_cast<size_t>(B) * 4,
                                 cudaMemcpyDeviceToHost, st_) != cudaSuccess)
    return FS_ERR_CUDA;
  return FS_OK;
}

fs_status fs_test_stall_loads(int on) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_test_stall = on != 0;
  return FS_OK;
}

fs_status fs_test_stalled_sample(const void *H, const void *W, int B, int d, int V,
                                 int32_t *out_idx, void *workspace, size_t workspace_bytes,
                                 fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, 1.0f, out_idx);
  if (s != FS_OK) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  g_test_no_loads = true;
  s = run_locked(fmms::kModeFlat, H, W, B, d, V, 1, 1.0f, 0, nullptr, 0, nullptr, out_idx,
                 nullptr, nullptr, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
  g_test_no_loads = false;
  return s;
}

fs_status fs_sample_shard_keys(const void *H, const void *W_shard, int B, int d, int V_shard,
                               int vocab_offset, int V_total, float temperature, uint64_t seed,
                               const uint64_t *row_seeds, uint32_t step, const uint32_t *mask_bits,
                               int64_t *out_keys, void *workspace, size_t workspace_bytes,
                               fs_stream_t stream) {
  fs_status s = validate(H, W_shard, B, d, V_shard, temperature, out_keys);
  if (s != FS_OK) return s;
  if (vocab_offset < 0 || (vocab_offset % fmms::kGranule) != 0 || V_total < 1 ||
      static_cast<int64_t>(vocab_offset) + V_shard > V_total)
    return FS_ERR_INVALID_ARG;
  ShardOpts opts;
  opts.vocab_offset = vocab_offset;
  opts.V_total = V_total;
  opts.out_keys = reinterpret_cast<long long *>(out_keys);
  std::lock_guard<std::mutex> lock(g_mu);
  return run_locked(fmms::kModeFlat, H, W_shard, B, d, V_shard, 1, temperature, seed, row_seeds,
                    step, mask_bits, reinterpret_cast<int32_t *>(out_keys), nullptr, nullptr,
                    workspace, workspace_bytes, static_cast<cudaStream_t>(stream), opts);
}

// ------------------------------------------- fused vocabulary-parallel exchange
// Longest wait fs_tp_wait accepts: one minute.
constexpr uint32_t kMaxTpWaitUs = 60u * 1000u * 1000u;

size_t fs_tp_area_bytes(void) { return fmms::kTpAreaBytes; }

fs_status fs_tp_area_create(void **area) {
  if (area == nullptr) return FS_ERR_INVALID_ARG;
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  *area = nullptr;
  if (fault_mode() == kFaultAlloc) return FS_ERR_CUDA;
  if (cudaMalloc(area, fmms::kTpAreaBytes) != cudaSuccess) return FS_ERR_CUDA;
  if (cudaMemset(*area, 0, fmms::kTpAreaBytes) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(*area);
    *area = nullptr;
    return FS_ERR_CUDA;
  }
  return FS_OK;
}

fs_status fs_tp_area_destroy(void *area) {
  if (area == nullptr) return FS_OK;
  return cudaFree(area) == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

fs_status fs_ipc_handle(const void *area, void *handle) {
  if (area == nullptr || handle == nullptr) return FS_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, const_cast<void *>(area)) != cudaSuccess) return FS_ERR_CUDA;
  static_assert(sizeof(h) == FS_IPC_HANDLE_BYTES, "IPC handle size");
  memcpy(handle, &h, sizeof h);
  return FS_OK;
}

fs_status fs_ipc_open(const void *handle, void **area) {
  if (handle == nullptr || area == nullptr) return FS_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof h);
  *area = nullptr;
  return cudaIpcOpenMemHandle(area, h, cudaIpcMemLazyEnablePeerAccess) == cudaSuccess
             ? FS_OK
             : FS_ERR_CUDA;
}

fs_status fs_ipc_close(void *area) {
  if (area == nullptr) return FS_OK;
  return cudaIpcCloseMemHandle(area) == cudaSuccess ? FS_OK : FS_ERR_CUDA;
}

fs_status fs_sample_tp(const void *H, const void *W_shard, int B, int d, int V_shard,
                       int vocab_offset, int V_total, float temperature, uint64_t seed,
                       const uint64_t *row_seeds, uint32_t step, const uint32_t *mask_bits,
                       void *const *areas, int world, uint32_t seq, void *workspace,
                       size_t workspace_bytes, fs_stream_t stream) {
  fs_status s = validate(H, W_shard, B, d, V_shard, temperature, areas);  // tokens go to the areas
  if (s != FS_OK) return s;
  if (B > fmms::kMaxBN) return FS_ERR_UNSUPPORTED;
  if (vocab_offset < 0 || (vocab_offset % fmms::kGranule) != 0 || V_total < 1 ||
      static_cast<int64_t>(vocab_offset) + V_shard > V_total)
    return FS_ERR_INVALID_ARG;
  if (areas == nullptr || world < 1 || world > fmms::kMaxTpWorld) return FS_ERR_INVALID_ARG;
  for (int r = 0; r < world; ++r)
    if (areas[r] == nullptr || (reinterpret_cast<uintptr_t>(areas[r]) & 255) != 0)
      return FS_ERR_INVALID_ARG;
  ShardOpts opts;
  opts.vocab_offset = vocab_offset;
  opts.V_total = V_total;
  opts.tp_world = world;
  opts.tp_seq = seq;
  opts.tp_areas = areas;
  std::lock_guard<std::mutex> lock(g_mu);
  return run_locked(fmms::kModeFlat, H, W_shard, B, d, V_shard, 1, temperature, seed, row_seeds,
                    step, mask_bits, nullptr, nullptr, nullptr, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream), opts);
}

fs_status fs_tp_wait(const void *area, int B, uint32_t seq, int32_t *out_idx,
                     uint32_t timeout_us, fs_stream_t stream) {
  if (area == nullptr || out_idx == nullptr || B < 1 || B > fmms::kMaxBN || timeout_us < 1 ||
      timeout_us > kMaxTpWaitUs)
    return FS_ERR_INVALID_ARG;
  if (launch_fault()) return FS_ERR_CUDA;
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  return fmms::launch_tp_wait(static_cast<fmms::TpArea *>(const_cast<void *>(area)), B, seq,
                              out_idx, timeout_us, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? FS_OK
             : FS_ERR_CUDA;
}

fs_status fs_tp_failed(const void *area, uint32_t *failed) {
  if (area == nullptr || failed == nullptr) return FS_ERR_INVALID_ARG;
  const fmms::TpArea *a = static_cast<const fmms::TpArea *>(area);
  return cudaMemcpy(failed, &a->failed, 4, cudaMemcpyDeviceToHost) == cudaSuccess ? FS_OK
                                                                                 : FS_ERR_CUDA;
}

fs_status fs_sample_multi(const void *H, const void *W, int B, int d, int V, int num_samples,
                          float temperature, uint64_t seed, const uint64_t *row_seeds,
                          uint32_t step, const uint32_t *mask_bits, int32_t *out_idx,
                          void *workspace, size_t workspace_bytes, fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, temperature, out_idx);
  if (s != FS_OK) return s;
  if (num_samples < 1 || num_samples > fmms::kMaxSamples) return FS_ERR_INVALID_ARG;
  ShardOpts opts;
  opts.num_samples = num_samples;
  std::lock_guard<std::mutex> lock(g_mu);
  return run_locked(fmms::kModeFlat, H, W, B, d, V, 1, temperature, seed, row_seeds, step,
                    mask_bits, out_idx, nullptr, nullptr, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream), opts);
}

size_t fs_workspace_bytes_multi(int B, int V, int num_samples) {
  if (B < 1 || V < 1 || num_samples < 1 || num_samples > fmms::kMaxSamples) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const Schedule sch = fmms::make_schedule(V, 1, sms);
  return static_cast<size_t>(fmms::workspace_bytes_for(B, 1, sch.num_ctas, num_samples));
}

fs_status fs_keys_to_tokens(const int64_t *keys, int B, int32_t *out_idx, fs_stream_t stream) {
  if (!keys || !out_idx || B < 1) return FS_ERR_INVALID_ARG;
  if (launch_fault()) return FS_ERR_CUDA;
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  return fmms::launch_keys_to_tokens(reinterpret_cast<const long long *>(keys), B, out_idx,
                                     static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FS_OK
             : FS_ERR_CUDA;
}

size_t fs_workspace_bytes(int B, int V, int G) {
  if (B < 1 || V < 1 || G < 0 || G > V) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const Schedule sch = fmms::make_schedule(V, G, sms);
  return static_cast<size_t>(fmms::workspace_bytes_for(B, sch.G, sch.num_ctas, 1, G >= 2));
}

fs_status fs_sample_topk(const void *H, const void *W, int B, int d, int V, int K,
                         float temperature, uint64_t seed, const uint64_t *row_seeds,
                         uint32_t step, const uint32_t *mask_bits, int32_t *out_idx,
                         float *logits, void *workspace, size_t workspace_bytes,
                         fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, temperature, out_idx);
  if (s != FS_OK) return s;
  if (!logits || K < 1) return FS_ERR_INVALID_ARG;
  ShardOpts opts;
  opts.top_k = K;
  std::lock_guard<std::mutex> lock(g_mu);
  return run_locked(fmms::kModeLogits, H, W, B, d, V, 1, temperature, seed, row_seeds, step,
                    mask_bits, out_idx, nullptr, logits, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream), opts);
}

size_t fs_workspace_bytes_summary(int B, int V_g) {
  if (B < 1 || V_g < 1) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const Schedule sch = fmms::make_schedule(V_g, 1, sms);
  return static_cast<size_t>(fmms::workspace_bytes_for(B, 1, sch.num_ctas, 1, true));
}

fs_status fs_summarize_group(const void *H, const void *W_g, int B, int d, int V_g,
                           int vocab_offset, int V_total, float temperature, uint64_t seed,
                           const uint64_t *row_seeds, uint32_t step, const uint32_t *mask_bits,
                           fs_group_summary *out_summary, void *workspace, size_t workspace_bytes,
                           fs_stream_t stream) {
  fs_status s = validate(H, W_g, B, d, V_g, temperature, out_summary);
  if (s != FS_OK) return s;
  if (vocab_offset < 0 || (vocab_offset % fmms::kGranule) != 0 || V_total < 1 ||
      static_cast<int64_t>(vocab_offset) + V_g > V_total)
    return FS_ERR_INVALID_ARG;
  ShardOpts opts;
  opts.vocab_offset = vocab_offset;
  opts.V_total = V_total;
  std::lock_guard<std::mutex> lock(g_mu);
  return run_locked(fmms::kModeGrouped, H, W_g, B, d, V_g, 1, temperature, seed, row_seeds, step,
                    mask_bits, nullptr, out_summary, nullptr, workspace, workspace_bytes,
                    static_cast<cudaStream_t>(stream), opts);
}

fs_status fs_merge_groups(const fs_group_summary *summaries, int G, int B, uint64_t seed,
                          const uint64_t *row_seeds, uint32_t step, int32_t *out_idx,
                          fs_stream_t stream) {
  if (!summaries || !out_idx || G < 1 || B < 1) return FS_ERR_INVALID_ARG;
  if (launch_fault()) return FS_ERR_CUDA;
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  return fmms::launch_merge_summaries(summaries, G, B, seed, row_seeds, step, out_idx,
                                      static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FS_OK
             : FS_ERR_CUDA;
}

fs_status fs_device_status(void *workspace, size_t workspace_bytes, fs_stream_t stream) {
  std::lock_guard<std::mutex> lock(g_mu);
  void *ws = workspace;
  size_t bytes = workspace_bytes;
  if (!ws) {
    DeviceState *st = nullptr;
    fs_status s = get_device(&st);
    if (s != FS_OK) return s;
    ws = st->ws;
    bytes = st->ws_bytes;
    if (!ws) return FS_OK;
  }
  if (bytes < static_cast<size_t>(fmms::kWsHeader)) return FS_ERR_WORKSPACE;
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st_) != cudaSuccess) return FS_ERR_CUDA;
  int err = 0;
  if (cudaMemcpy(&err, ws, sizeof err, cudaMemcpyDeviceToHost) != cudaSuccess) return FS_ERR_CUDA;
  if (err == 0) return FS_OK;
  if (cudaMemset(ws, 0, bytes) != cudaSuccess) return FS_ERR_CUDA;
  return err == fmms::kErrBounds ? FS_ERR_DEVICE_BOUNDS : FS_ERR_DEVICE_TIMEOUT;
}

const char *fs_status_string(fs_status status) {
  switch (status) {
    case FS_OK: return "FS_OK";
    case FS_ERR_INVALID_ARG: return "FS_ERR_INVALID_ARG";
    case FS_ERR_UNSUPPORTED: return "FS_ERR_UNSUPPORTED";
    case FS_ERR_CUDA: return "FS_ERR_CUDA";
    case FS_ERR_WORKSPACE: return "FS_ERR_WORKSPACE";
    case FS_ERR_DEVICE_TIMEOUT: return "FS_ERR_DEVICE_TIMEOUT";
    case FS_ERR_DEVICE_BOUNDS: return "FS_ERR_DEVICE_BOUNDS";
  }
  return "FS_ERR_UNKNOWN";
}

fs_status fs_philox4x32_10(const uint32_t *ctr, const uint32_t *key, uint32_t *out, int64_t n,
                           fs_stream_t stream) {
  if (n < 0 || (n > 0 && (!ctr || !key || !out))) return FS_ERR_INVALID_ARG;
  if (launch_fault()) return FS_ERR_CUDA;
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  return fmms::launch_philox_test(ctr, key, out, n, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FS_OK
             : FS_ERR_CUDA;
}

fs_status fs_gumbel(const uint32_t *r, float *g, int64_t n, fs_stream_t stream) {
  if (n < 0 || (n > 0 && (!r || !g))) return FS_ERR_INVALID_ARG;
  if (launch_fault()) return FS_ERR_CUDA;
  DeviceState *st = nullptr;
  fs_status s = get_device(&st);
  if (s != FS_OK) return s;
  return fmms::launch_gumbel_test(r, g, n, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FS_OK
             : FS_ERR_CUDA;
}

fs_status fs_set_partial_merge(int policy) {
  if (policy < -1 || policy > 1) return FS_ERR_INVALID_ARG;
  read_force_path();
  std::lock_guard<std::mutex> lock(g_mu);
  g_merge_policy = policy;
  return FS_OK;
}

fs_status fs_test_inject_fault(int kind, int *previous) {
  if (kind < -1 || kind > kFaultLaunch) return FS_ERR_INVALID_ARG;
  const int before = fault_mode();
  if (previous) *previous = before;
  if (kind >= 0) g_fault.store(kind, std::memory_order_relaxed);
  return FS_OK;
}

fs_status fs_get_policies(int *cta_pairs, int *partial_merge, int *programmatic,
                          int *unfused, int *two_kernel_reduce) {
  read_force_path();
  std::lock_guard<std::mutex> lock(g_mu);
  if (cta_pairs) *cta_pairs = g_pair_policy;
  if (partial_merge) *partial_merge = g_merge_policy;
  if (programmatic) *programmatic = g_pdl_policy;
  if (unfused) *unfused = g_force_unfused ? 1 : 0;
  if (two_kernel_reduce) *two_kernel_reduce = g_two_kernel_reduce ? 1 : 0;
  return FS_OK;
}

fs_status fs_set_programmatic_launch(int on) {
  if (on < 0 || on > 1) return FS_ERR_INVALID_ARG;
  read_force_path();
  std::lock_guard<std::mutex> lock(g_mu);
  g_pdl_policy = on;
  return FS_OK;
}

fs_status fs_set_cta_pairs(int policy) {
  if (policy < -1 || policy > 1) return FS_ERR_INVALID_ARG;
  read_force_path();
  std::lock_guard<std::mutex> lock(g_mu);
  g_pair_policy = policy;
  return FS_OK;
}

fs_status fs_plan_tiles(int V, int G, int num_sms, int cta, int32_t *tiles, int max_tiles,
                        int *ntiles, int *num_ctas_out) {
  if (V < 1 || G < 0 || G > V || num_sms < 1 || !ntiles) return FS_ERR_INVALID_ARG;
  const Schedule sch = fmms::make_schedule(V, G, num_sms);
  if (num_ctas_out) *num_ctas_out = sch.num_ctas;
  if (cta < 0 || cta >= sch.num_ctas) return FS_ERR_INVALID_ARG;
  fmms::TileIter it(sch, cta);
  fmms::Tile t;
  int n = 0;
  while (it.next(t)) {
    if (tiles && n < max_tiles) {
      tiles[5 * n + 0] = t.start;
      tiles[5 * n + 1] = t.lo;
      tiles[5 * n + 2] = t.hi;
      tiles[5 * n + 3] = t.slot;
      tiles[5 * n + 4] = t.last;
    }
    ++n;
  }
  *ntiles = n;
  return FS_OK;
}

fs_status fs_plan_tiles_merged(int V, int G, int num_sms, int cta, int32_t *tiles,
                               int max_tiles, int *ntiles, int *merges) {
  if (V < 1 || G < 0 || G > V || num_sms < 1 || !ntiles) return FS_ERR_INVALID_ARG;
  const Schedule sch = fmms::make_schedule(V, G, num_sms);
  if (merges) *merges = merge_rule(sch) ? 1 : 0;
  if (cta < 0 || cta >= sch.num_ctas) return FS_ERR_INVALID_ARG;
  fmms::TileIter it(sch, cta, 1);
  fmms::Tile t;
  int n = 0;
  while (it.next(t)) {
    if (tiles && n < max_tiles) {
      const int32_t row[8] = {t.start, t.lo, t.hi, t.slot, t.last, t.pstart, t.plo, t.phi};
      memcpy(tiles + 8 * n, row, sizeof row);
    }
    ++n;
  }
  *ntiles = n;
  return FS_OK;
}

fs_status fs_plan_batch(int B, int kind, int *launches, int *batch_tile, int *cta_pairs) {
  if (B < 1 || kind < 0 || kind > 2 || !launches) return FS_ERR_INVALID_ARG;
  read_force_path();
  const int mode = kind == 1 ? fmms::kModeGrouped : kind == 2 ? fmms::kModeLogits : fmms::kModeFlat;
  const int first = fmms::imin(fmms::kMaxBN, B);
  const int BN = fmms::fmms_batch_tile(first);
  *launches = (B + fmms::kMaxBN - 1) / fmms::kMaxBN;
  if (batch_tile) *batch_tile = BN;
  if (cta_pairs) {
    std::lock_guard<std::mutex> lock(g_mu);
    *cta_pairs = use_pairs(mode, BN) ? 1 : 0;
  }
  return FS_OK;
}

fs_status fs_plan_group_ctas(int V, int G, int num_sms, int g, int *first, int *last) {
  if (V < 1 || G < 1 || G > V || num_sms < 1 || g < 0 || g >= G || !first || !last)
    return FS_ERR_INVALID_ARG;
  const Schedule sch = fmms::make_schedule(V, G, num_sms);
  *first = fmms::cta_of(fmms::group_begin(g, V, G), sch);
  *last = fmms::cta_of(fmms::group_begin(g + 1, V, G) - 1, sch);
  return FS_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free entry point: scratch in a fixed device array of this file.
// ---------------------------------------------------------------------------
namespace {

// Status word + ticket (256 bytes) and packed keys of up to 256 rows.
constexpr size_t kNoAllocScratchBytes = fmms::kWsHeader + fmms::kWsKeys;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on each device (null until looked up).
// In host code the array's name is only a host-side stand-in.
void *g_noalloc_addr[kMaxDevices];

}  // namespace

extern "C" fs_status fs_sample_noalloc(const void *H, const void *W, int B, int d, int V,
                                       float temperature, uint64_t seed,
                                       const uint64_t *row_seeds, uint32_t step,
                                       const uint32_t *mask_bits, int32_t *out_idx,
                                       fs_stream_t stream) {
  fs_status s = validate(H, W, B, d, V, temperature, out_idx);
  if (s != FS_OK) return s;
  if (B > fmms::kMaxBN) return FS_ERR_UNSUPPORTED;  // keys for at most 256 rows
  if (static_cast<size_t>(fmms::workspace_bytes_for(B, 1, 1)) > kNoAllocScratchBytes)
    return FS_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FS_ERR_CUDA;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_noalloc_addr[dev] == nullptr) {
      void *p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return FS_ERR_CUDA;
      g_noalloc_addr[dev] = p;
    }
    scratch = g_noalloc_addr[dev];
  }
  // Everything after the status word starts at zero (the ticket and keys are
  // left zeroed by a completed call, but not by one that gave up on a
  // bounded wait); the status word keeps a recorded timeout until
  // fs_noalloc_status reads and clears it.
  if (launch_fault()) return FS_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<char *>(scratch) + 4, 0, kNoAllocScratchBytes - 4, st) !=
      cudaSuccess)
    return FS_ERR_CUDA;
  return run(fmms::kModeFlat, H, W, B, d, V, 1, temperature, seed, row_seeds, step, mask_bits,
             out_idx, nullptr, nullptr, scratch, kNoAllocScratchBytes, st);
}

extern "C" fs_status fs_noalloc_status(fs_stream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FS_ERR_CUDA;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    scratch = g_noalloc_addr[dev];
  }
  if (scratch == nullptr) return FS_OK;  // no call on this device yet
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FS_ERR_CUDA;
  int err = 0;
  if (cudaMemcpy(&err, scratch, sizeof err, cudaMemcpyDeviceToHost) != cudaSuccess)
    return FS_ERR_CUDA;
  if (err == 0) return FS_OK;
  if (cudaMemset(scratch, 0, kNoAllocScratchBytes) != cudaSuccess) return FS_ERR_CUDA;
  return err == fmms::kErrBounds ? FS_ERR_DEVICE_BOUNDS : FS_ERR_DEVICE_TIMEOUT;
}
