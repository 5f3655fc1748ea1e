// fmms_common.cuh -- host/device definitions shared by the FMMS kernels and
// the C ABI: tile geometry, the split-V schedule, kernel parameters and the
// packed (score, token) key used by every reduction.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define FS_HD __host__ __device__ __forceinline__
#else
#define FS_HD inline
#endif

namespace fmms {

// Tile geometry (swap-AB orientation: vocabulary rows on the MMA M axis and
// TMEM lanes, batch rows on the MMA N axis and TMEM columns).
constexpr int kTileM = 128;   // vocabulary rows per tile (tcgen05 M)
constexpr int kBlockK = 64;   // K elements per pipeline stage: one 128-byte swizzle row
constexpr int kGranule = 8;   // vocabulary granule of the per-CTA split: one 8-row swizzle atom
constexpr int kMaxBN = 256;   // batch rows per launch (tcgen05 N limit)

// The batch tiles the kernels are built for: every multiple of 16 rows up to
// 256 (tcgen05 N with M = 128 or, on CTA pairs, M = 256; 8-row halves).
#define FMMS_FOR_EACH_BN(X) \
  X(16) X(32) X(48) X(64) X(80) X(96) X(112) X(128) X(144) X(160) X(176) X(192) X(208) X(224) \
  X(240) X(256)
constexpr int kNumEpiWarps = 16;  // four per TMEM lane quarter
constexpr int kThreads = 32 * (2 + kNumEpiWarps);  // TMA warp + MMA warp + epilogue
constexpr int kEpiThreads = 32 * kNumEpiWarps;

FS_HD int imin(int a, int b) { return a < b ? a : b; }
FS_HD int imax(int a, int b) { return a > b ? a : b; }

// ---------------------------------------------------------------------------
// Debug build (compiled with -DFS_DEBUG, libfmms_debug.so): device-side bounds
// checks on the kernels' global, shared and tensor memory indices.  A check
// that fails records kErrBounds in the call's status word (the first error
// recorded wins) and the access is skipped; nothing traps, so the context
// stays usable and the host reads the error with fs_device_status.  In the
// release build every check is the constant true and compiles away.
// ---------------------------------------------------------------------------
constexpr int kErrBounds = 6;
#if defined(FS_DEBUG) && defined(__CUDACC__)
__device__ __forceinline__ bool dbg_in_bounds(int *err, long long i, long long n) {
  if (i >= 0 && i < n) return true;
  if (err != nullptr) atomicCAS(err, 0, kErrBounds);
  return false;
}
#define FS_IN_BOUNDS(err, i, n) ::fmms::dbg_in_bounds((err), (long long)(i), (long long)(n))
#else
#define FS_IN_BOUNDS(err, i, n) true
#endif

// ---------------------------------------------------------------------------
// Split-V schedule.  The vocabulary is cut into ceil(V/8) granules; CTA c of
// num_ctas owns granules [floor(c n / C), floor((c+1) n / C)), so every CTA
// streams the same number of W rows to within one granule.  Group g of G
// covers [floor(g V / G), floor((g+1) V / G)).  A CTA's range is cut at group
// boundaries into segments; each segment is walked in 128-row tiles (256 on
// CTA pairs) starting at its first token rounded down to a multiple of 8 (rows
// before the segment are loaded but ignored), its partial tile first.
// Segment (c, g) owns partial slot c + g, which is unique because c and g
// never both stay put from one segment to the next.
// ---------------------------------------------------------------------------
struct Schedule {
  int V;
  int G;          // number of groups (1 = flat)
  int num_ctas;   // schedule units: CTAs, or CTA pairs in pair mode
  int ngran;      // ceil(V / 8)
  int tile_rows;  // vocabulary rows per tile: 128, or 256 for a CTA pair
};

FS_HD Schedule make_schedule(int V, int G, int num_sms) {
  Schedule s;
  s.V = V;
  s.G = G < 1 ? 1 : G;
  s.ngran = (V + kGranule - 1) / kGranule;
  s.num_ctas = imin(num_sms, s.ngran);
  s.tile_rows = kTileM;
  return s;
}

FS_HD int group_begin(int g, int V, int G) { return (int)(((int64_t)g * V) / G); }

// The group containing token v: the largest g with floor(g V / G) <= v.
FS_HD int group_of(int v, int V, int G) {
  return (int)((((int64_t)v + 1) * G - 1) / V);
}

FS_HD int cta_begin(int c, const Schedule &s) {
  int64_t gran = ((int64_t)c * s.ngran) / s.num_ctas;
  int64_t v = gran * kGranule;
  return v < s.V ? (int)v : s.V;
}

// The CTA whose range contains token v.
FS_HD int cta_of(int v, const Schedule &s) {
  int64_t q = v / kGranule;
  return (int)(((q + 1) * s.num_ctas - 1) / s.ngran);
}

struct Tile {
  int start;  // first vocabulary row of the tile (multiple of 8)
  int lo;     // first valid row
  int hi;     // one past the last valid row (hi - start <= tile rows)
  int slot;   // partial slot of the segment
  int last;   // 1 on the last tile of a segment
  // Merged partial: an 8-row partial tile [pstart, pstart + 8) (valid rows
  // [plo, phi)) multiplied in the same stages as this whole tile, sharing
  // its H loads, into an accumulator of its own.  pstart < 0: none.
  int pstart, plo, phi;
};

// The merged partial of a tile as a tile of its own.
FS_HD Tile partial_of(const Tile &t) {
  Tile p = t;
  p.start = t.pstart;
  p.lo = t.plo;
  p.hi = t.phi;
  p.pstart = -1;
  return p;
}

// The 128-row half of a 256-row pair tile that CTA `rank` of the pair
// multiplies; hi <= lo when the half holds no valid row.
FS_HD Tile pair_half(const Tile &t, int rank) {
  Tile h = t;
  h.start = t.start + rank * kTileM;
  h.lo = imax(t.lo, h.start);
  h.hi = imin(t.hi, h.start + kTileM);
  return h;
}

// Walks the tiles of one CTA.  All three kernel roles and the host-side
// schedule query run this same code.
struct TileIter {
  int V, G, cta, cta_hi, rows;
  int v;       // first token of the current segment
  int seg_hi;  // end of the current segment
  int t;       // start of the next tile
  int len;     // rows of the next tile
  int slot;
  int merge;   // merge a segment's 8-row partial tile into its first whole tile

  FS_HD TileIter(const Schedule &s, int c, int merge_partial = 0) {
    merge = merge_partial;
    V = s.V;
    G = s.G;
    rows = s.tile_rows;
    cta = c;
    v = cta_begin(c, s);
    cta_hi = cta_begin(c + 1, s);
    seg_hi = v;
    t = v;
    len = rows;
    slot = c;
  }

  // A segment's partial tile comes first: its remainder rows, rounded up to a
  // multiple of 8, then whole tiles (the last may lack up to 7 rows).  The MMA
  // loop of a partial tile costs as much as a whole tile's; run first it
  // overlaps the other CTAs' streaming, run last it would be a tail with HBM
  // idle.  With `merge`, an 8-row partial tile followed by a whole tile is
  // returned with it (pstart), so that both share one pass over H.
  FS_HD bool next(Tile &tile) {
    tile.pstart = -1;
    tile.plo = tile.phi = 0;
    if (t >= seg_hi) {
      v = seg_hi;
      if (v >= cta_hi) return false;
      int g = G > 1 ? group_of(v, V, G) : 0;
      int gend = G > 1 ? group_begin(g + 1, V, G) : V;
      seg_hi = imin(cta_hi, gend);
      slot = cta + g;
      t = v & ~(kGranule - 1);
      const int rem = (seg_hi - t) % rows;
      len = rem == 0 ? rows : (rem + kGranule - 1) & ~(kGranule - 1);
    }
    if (merge && len == kGranule && t + len < seg_hi) {
      tile.pstart = t;
      tile.plo = imax(t, v);
      tile.phi = imin(t + len, seg_hi);
      t += len;
      len = rows;
    }
    tile.start = t;
    tile.lo = imax(t, v);
    tile.hi = imin(t + len, seg_hi);
    tile.slot = slot;
    t += len;
    len = rows;
    tile.last = (t >= seg_hi) ? 1 : 0;
    return true;
  }
};

// ---------------------------------------------------------------------------
// Packed (score, token) key.  Unsigned 64-bit order on
//   (order_bits(s) << 32) | (0xFFFFFFFF - v)
// is "larger score first, then smaller token", the tie rule of every argmax
// here.  A key whose high word is 0 means "no candidate" (a masked or
// out-of-range entry): every finite or infinite score maps to a nonzero
// high word.
// ---------------------------------------------------------------------------
FS_HD uint32_t order_bits(uint32_t f) {
  // negative: flip every bit; non-negative: set the sign bit
  return f ^ (static_cast<uint32_t>(static_cast<int32_t>(f) >> 31) | 0x80000000u);
}
FS_HD uint32_t order_bits_inv(uint32_t o) {
  return (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
}
FS_HD uint64_t pack_key(uint32_t score_bits, int v) {
  return ((uint64_t)order_bits(score_bits) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)v);
}
FS_HD bool key_valid(uint64_t k) { return (k >> 32) != 0; }
FS_HD int key_token(uint64_t k) { return key_valid(k) ? (int)(0xFFFFFFFFu - (uint32_t)k) : -1; }
FS_HD uint32_t key_score_bits(uint64_t k) { return order_bits_inv((uint32_t)(k >> 32)); }

// Per-(slot, row) partial of the grouped kernel.
struct __align__(16) GroupPartial {
  unsigned long long key;  // packed best (score, token)
  float m;                 // max of allowed x in the segment (-inf if none)
  float sum;               // sum of exp(x - m) over allowed x
};

enum Mode { kModeFlat = 0, kModeGrouped = 1, kModeLogits = 2 };

// Fused vocabulary-parallel exchange.  Each rank of a tensor-parallel group
// owns one exchange area in its own device memory; every rank's kernel maps
// all of them (its own and its peers', over NVLink).  Calls are numbered by a
// sequence number seq, the same on every rank; seq & 1 selects the half of
// the area a call uses, so a rank one call ahead never touches the half
// still being decoded.  Per call, the last CTA of each rank's kernel raises
// every area's keys to its rows' packed maxima, then counts itself in every
// area's arrivals; the arrival that completes an area decodes its keys into
// its tokens, clears the keys and the count, and sets its flag to seq + 1.
// No sampling kernel waits for another: the stream that needs the tokens runs
// a small kernel that polls the flag, for a bounded time, and copies them.
constexpr int kMaxTpWorld = 16;
struct TpArea {
  unsigned int arrivals[2];  // ranks counted in, per parity
  unsigned int err[2];       // set by a rank whose kernel recorded a device error
  unsigned int flag;         // seq + 1 of the last call decoded into tokens
  unsigned int failed;       // seq + 1 of the last call decoded with an error
  unsigned int pad[2];
  unsigned long long keys[2][kMaxBN];
  int tokens[2][kMaxBN];     // -1 for every row of a call with an error
};
constexpr size_t kTpAreaBytes = (sizeof(TpArea) + 255) / 256 * 256;

struct FmmsParams {
  int B;            // rows in this launch (<= BN)
  int b_off;        // global index of this launch's row 0 (noise, mask, seeds)
  int d;
  int V;
  int G;
  int num_ctas;
  int ngran;
  int nk;           // ceil(d / 64) pipeline stages per tile
  float inv_temp;
  uint32_t step;
  uint64_t seed;
  const uint64_t *row_seeds;   // [global rows] or null
  const uint32_t *mask;        // [global rows][mask_words] or null
  int mask_words;
  int32_t *out_idx;            // [B] (already offset to this launch)
  unsigned long long *keys;    // workspace [B]: running packed maxima (flat)
  unsigned int *ticket;        // workspace: CTAs finished (flat)
  int *err;                    // workspace: device status word
  GroupPartial *partials;      // workspace [slots][B] (grouped)
  unsigned long long *gkeys;   // workspace [G][B] published per-group maxima, or null
  float *logits;               // [B][V] (logits mode; already offset)
  int test_no_loads;           // test hook: the producer issues no loads, so waits time out
  int vocab_offset;            // global token index of W row 0 (a vocabulary shard), % 8 == 0
  long long *out_keys;         // if set: per-row packed keys XOR 2^63 instead of tokens
  int num_samples;             // samples per row (flat mode), 1..kMaxSamples
  // H arriving while the kernel runs (fs_sample_host): 64-wide K sub-block s
  // of H may be loaded once h_ready[s / h_chunk_subs] == h_epoch.  Null: H is
  // complete when the kernel starts.
  const uint32_t *h_ready;
  uint32_t h_epoch;
  int h_chunk_subs;
  // Fused vocabulary-parallel exchange (flat mode): tp_world > 0 replaces the
  // token output; tp_area[r] is rank r's exchange area, mapped here.
  int tp_world;
  uint32_t tp_seq;
  TpArea *tp_area[kMaxTpWorld];
  // 1: launched as a programmatic dependent of the grid ahead in the stream
  // (may start before it ends; H loads and workspace accesses wait for it).
  int pdl;
  // Flat mode: 1 leaves the published keys for a second kernel to decode
  // (the two-kernel reduction, an A/B alternative to the last-CTA ticket).
  int no_ticket;
  // Extents the debug build's bounds checks compare against (entries, not
  // bytes): rows of row_seeds and mask (the whole call), packed keys in the
  // workspace, partial records and published group maxima, and tokens (or
  // keys) and logits this launch may write.
  int rows_total;
  int keys_cap;
  long long partials_cap;
  long long gkeys_cap;
  int out_cap;
  long long logits_cap;
};

// Workspace layout (bytes), fixed so that calls of different kinds can share
// one workspace: [0, 256) status word and ticket; [256, 256 + 64 * 2048)
// packed keys [sample][256 rows], of which a flat call uses (and needs) only
// its samples' part; then, grouped only, the partials [slots][rows] and, for
// G <= kMaxPublishedGroups, the published per-group maxima [G][rows] that
// sharpen the exact-score filter.  Where the partials and maxima lie depends
// on (B, G), so one call's published maxima may sit where an earlier call
// kept partials: every completed call therefore leaves all it used zeroed
// (the merge kernel zeroes each partial it reads and each published maximum),
// and every call finds its published maxima at zero.
constexpr int kWsHeader = 256;
constexpr int kWsKeys = 8 * kMaxBN;
constexpr int kMaxPublishedGroups = 4096;
constexpr int kMaxSamples = 64;
constexpr int kWsKeysRegion = kMaxSamples * kWsKeys;

// Partial slots: num_ctas + G - 1 for single CTAs; a CTA pair writes two
// slots per (pair, group) segment, 2 (pairs + G - 1) in all, and a launch
// never has more pairs than the single-CTA schedule has CTAs.
FS_HD int64_t ws_partials_bytes(int B, int G, int num_ctas) {
  const int64_t rows = B < kMaxBN ? B : kMaxBN;
  return 2 * (int64_t)(num_ctas + G - 1) * rows * (int64_t)sizeof(GroupPartial);
}

FS_HD int64_t ws_gkeys_bytes(int B, int G) {
  const int64_t rows = B < kMaxBN ? B : kMaxBN;
  return G <= kMaxPublishedGroups ? (int64_t)G * rows * 8 : 0;
}

// Bytes of workspace for a flat call with `samples` samples, or a grouped call
// (grouped = true) with G >= 1 groups.
FS_HD int64_t workspace_bytes_for(int B, int G, int num_ctas, int samples = 1,
                                  bool grouped = false) {
  const int64_t bytes =
      grouped ? (int64_t)kWsHeader + kWsKeysRegion + ws_partials_bytes(B, G, num_ctas) +
                    ws_gkeys_bytes(B, G)
              : (int64_t)kWsHeader + (int64_t)kWsKeys * (samples < 1 ? 1 : samples);
  return (bytes + 255) / 256 * 256;
}

}  // namespace fmms
