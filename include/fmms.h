/*
 * fmms.h -- C ABI of the FlashSampling fused matmul-sample (FMMS) library for
 * NVIDIA B200 (sm_100a), libfmms.so.
 *
 * The method (FlashSampling: Fast and Memory-Efficient Exact Sampling,
 * Ruiz et al., arXiv:2603.15854, abstract): the LM-head logits
 * l = h W^T are computed tile by tile on chip, Gumbel noise is added, only
 * one maximiser per row and per vocabulary tile is kept, and a small
 * reduction over tiles returns one sampled token per row.  The B x V logits
 * tensor never reaches HBM.  It is exact because argmax decomposes over a
 * partition of the vocabulary (Gumbel-Max theorem, readus.org page, section
 * "Gumbel Max Trick").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  H      hidden states, bf16 [B, d], row-major (row b is contiguous).
 *  W      LM-head weight, bf16 [V, d], row-major (the nn.Linear layout).
 *         Both base addresses must be 16-byte aligned and d % 8 == 0 (rows
 *         are read by TMA with 16-byte strides).  B >= 1, V >= 1.
 *  temperature  T > 0 and finite; scores are x = l / T.  The Gumbel noise is
 *         not scaled by T (readus.org page, "API": temperature is an argument
 *         of the sampling call).
 *  mask_bits  optional per-row vocab bitmask, uint32 [B][ceil(V/32)]: bit
 *         (v & 31) of word [b][v >> 5] is 1 when token v is allowed.
 *         Forbidden tokens get score -inf before the noise, so they are never
 *         sampled (readus.org page, "Top-K and masking").  NULL = all allowed.
 *  seed, row_seeds, step  the noise for (row b, token v) is word (v & 3) of
 *         Philox4x32-10 (Salmon et al., SC'11) with key = (k lo32, k hi32),
 *         k = row_seeds[b] if row_seeds is non-NULL else seed, and counter
 *         (v >> 2, b, step, 0).  The noise is therefore a pure function of
 *         (seed, step, row, token): the same call gives the same tokens on
 *         any device, stream or tiling (readus.org page, "seed management").
 *  noise  g = -log(-log u), u = (r + 1) / (2^32 + 1) for the noise word r
 *         (readus.org page, "floating point precision"); u never reaches 0
 *         or 1, so g is always finite.
 *  out_idx  int32 [B]: the sampled token of each row, the smallest v
 *         attaining max_v (x[b,v] + g[b,v]); -1 when every token of the row is
 *         masked (a per-row result, not an error).
 *  stream  a cudaStream_t passed as an opaque pointer; NULL is the legacy
 *         default stream.  Every entry point is asynchronous on `stream`
 *         unless stated otherwise: it validates its arguments, enqueues its
 *         kernels and returns.  Output buffers are valid once the stream has
 *         reached that point; the caller keeps every buffer alive until then.
 *  memory  unless stated otherwise every array pointer is a DEVICE pointer on
 *         the current device, owned by the caller.  The library keeps no
 *         pointer past the call.
 *  workspace  entry points that take (workspace, workspace_bytes) use the
 *         caller's device buffer of at least fs_workspace_bytes(B, V, G) bytes,
 *         256-byte aligned, which must be zero-filled before its first use
 *         (cudaMemset).  Every call that completes leaves every byte it used
 *         zeroed again (status, ticket, per-row keys, the grouped calls'
 *         partials and published maxima), so one workspace may serve calls of
 *         any kind and size it is large enough for, whatever part of it each
 *         call lays out where.  Calls that share a workspace must be ordered on one stream.  With
 *         workspace == NULL the library uses its own per-device workspace,
 *         allocated on first use; such calls must not run concurrently on
 *         different streams.
 *  errors  argument errors are detected on the host before anything is
 *         enqueued and returned synchronously; launch failures return
 *         FS_ERR_CUDA.  A device-side wait that exceeds its time limit (about
 *         one second) makes the kernel record FS_ERR_DEVICE_TIMEOUT in the
 *         workspace and exit early; fs_device_status() reports it.
 */
#ifndef FMMS_H_
#define FMMS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FS_OK = 0,
  FS_ERR_INVALID_ARG = 1,    /* a pointer, size, alignment or value is invalid */
  FS_ERR_UNSUPPORTED = 2,    /* no sm_100 device, or a shape outside the supported range */
  FS_ERR_CUDA = 3,           /* a CUDA runtime/driver call or a launch failed */
  FS_ERR_WORKSPACE = 4,      /* the workspace is too small or misaligned */
  FS_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up on a bounded wait (see fs_device_status) */
  FS_ERR_DEVICE_BOUNDS = 6   /* debug build only: a device-side bounds check failed and the
                                access was skipped (see fs_device_status) */
} fs_status;

/* A cudaStream_t, passed without the CUDA headers. */
typedef void *fs_stream_t;

/* Per-(row, group) summary of the grouped sampler. */
typedef struct {
  float max_score; /* max over the group of x + g (-inf if the group is fully masked) */
  int32_t argmax;  /* the token attaining it (smallest index on ties), -1 if none */
  float lse;       /* log sum_{v in group, allowed} exp(x[v]), -inf if none */
} fs_group_summary;

/* Flat FMMS sample of B rows with one scalar seed and the library-owned
 * workspace (fused LM-head matmul + temperature + optional mask + Gumbel
 * noise + per-tile argmax + cross-tile reduction; abstract of the paper).
 * One kernel launch for B <= 256; larger B is processed in chunks of 256
 * rows.  Not safe for concurrent calls on different streams. */
fs_status fs_sample(const void *H, const void *W, int B, int d, int V,
                    float temperature, uint64_t seed, uint32_t step,
                    const uint32_t *mask_bits, int32_t *out_idx,
                    fs_stream_t stream);

/* fs_sample with optional per-row seeds (row_seeds: device uint64 [B] or
 * NULL) and an optional caller workspace (see "workspace" above). */
fs_status fs_sample_ex(const void *H, const void *W, int B, int d, int V,
                       float temperature, uint64_t seed,
                       const uint64_t *row_seeds, uint32_t step,
                       const uint32_t *mask_bits, int32_t *out_idx,
                       void *workspace, size_t workspace_bytes,
                       fs_stream_t stream);

/* Grouped sampling (Group-Gumbel-Max; readus.org page, section "Group Gumbel
 * Max"; abstract: grouped variants are exact by hierarchical factorisation
 * of the categorical distribution).  The vocabulary is split into G
 * contiguous groups, group g = [floor(g V / G), floor((g+1) V / G)),
 * 1 <= G <= V.  Per row and group the fused kernel keeps (max x + g, argmax,
 * lse = log sum exp(x) over allowed tokens); a merge kernel then picks
 * g* = argmax_g (lse_g + gumbel_g), where gumbel_g uses the noise word
 * (g & 3) of Philox(key, (g >> 2, b, step, 1)), and returns the argmax of
 * group g*.  The result equals flat sampling in distribution (not bitwise).
 * out_summary: optional device fs_group_summary [B][G] (NULL to skip). */
fs_status fs_sample_grouped(const void *H, const void *W, int B, int d, int V,
                            int G, float temperature, uint64_t seed,
                            const uint64_t *row_seeds, uint32_t step,
                            const uint32_t *mask_bits, int32_t *out_idx,
                            fs_group_summary *out_summary, void *workspace,
                            size_t workspace_bytes, fs_stream_t stream);

/* Unfused two-kernel mode, kept to measure the HBM traffic the fused kernel
 * saves: the matmul writes fp32 logits l (before temperature) to
 * logits [B][V] (device, caller-owned, row-major), then a second kernel
 * applies temperature, mask and noise and reduces to out_idx.  Returns the
 * same tokens as fs_sample_ex up to fp32 rounding of the logits. */
fs_status fs_sample_unfused(const void *H, const void *W, int B, int d, int V,
                            float temperature, uint64_t seed,
                            const uint64_t *row_seeds, uint32_t step,
                            const uint32_t *mask_bits, int32_t *out_idx,
                            float *logits, void *workspace,
                            size_t workspace_bytes, fs_stream_t stream);

/* Several samples per row from one pass over W (readus.org page, API: the
 * number of samples is an argument of the sampling call).  Sample k of row b
 * uses token noise with counter tag 2k, so the samples are independent exact
 * draws from softmax(l/T) (with replacement) and sample 0 is the fs_sample_ex
 * token.  out_idx is device int32 [B][num_samples] (row-major), 1 <= num_samples
 * <= 64.  The workspace needs fs_workspace_bytes_multi(B, V, num_samples)
 * bytes; other arguments as fs_sample_ex. */
fs_status fs_sample_multi(const void *H, const void *W, int B, int d, int V,
                          int num_samples, float temperature, uint64_t seed,
                          const uint64_t *row_seeds, uint32_t step,
                          const uint32_t *mask_bits, int32_t *out_idx,
                          void *workspace, size_t workspace_bytes,
                          fs_stream_t stream);

/* Online grouped sampling, one group at a time (readus.org page, "Group
 * Gumbel Max": only one group of the vocabulary needs to be on chip at a
 * time, its "captain" kept and the rest discarded; abstract: grouped variants
 * for online settings are exact by hierarchical factorisation).  W_g holds
 * rows [vocab_offset, vocab_offset + V_g) of a head with V_total rows
 * (vocab_offset % 8 == 0), delivered separately from the other groups.
 * Writes per row b the group's summary (max x + g, its global token, lse of
 * the allowed x = l / T) to out_summary[b] (device fs_group_summary [B]).
 * Token noise, mask and indices are global, as in fs_sample_grouped.  The
 * workspace needs fs_workspace_bytes_summary(B, V_g) bytes. */
fs_status fs_summarize_group(const void *H, const void *W_g, int B, int d,
                           int V_g, int vocab_offset, int V_total,
                           float temperature, uint64_t seed,
                           const uint64_t *row_seeds, uint32_t step,
                           const uint32_t *mask_bits,
                           fs_group_summary *out_summary, void *workspace,
                           size_t workspace_bytes, fs_stream_t stream);

/* Merges G group summaries (device fs_group_summary [G][B]: the summaries of
 * group g at [g][0..B)) by Group-Gumbel-Max: g* = argmax_g (lse_g + gumbel_g)
 * with gumbel_g from noise word (g & 3) of Philox(key, (g >> 2, b, step, 1)),
 * ties to the smaller g; out_idx[b] = the argmax of group g*, or -1 when every
 * group of the row is fully masked.  With the contiguous groups
 * [floor(g V/G), floor((g+1) V/G)) this is fs_sample_grouped (the group lse
 * may differ in the last fp32 bits, which can change g* only at near ties). */
fs_status fs_merge_groups(const fs_group_summary *summaries, int G, int B,
                          uint64_t seed, const uint64_t *row_seeds,
                          uint32_t step, int32_t *out_idx, fs_stream_t stream);

/* One vocabulary shard of a tensor-parallel LM head (readus.org page,
 * "distributed FlashSampling": each GPU is one group of the vocabulary and
 * contributes only its winning index and score; abstract: the argmax
 * decomposes over any partition).  W_shard holds rows
 * [vocab_offset, vocab_offset + V_shard) of a head with V_total rows;
 * vocab_offset must be a multiple of 8.  Noise, mask and token indices are
 * global, so the shard's candidates are exactly those of the full head.
 * Writes, per row, the shard's best (score, global token) as a packed key in
 * out_keys (device int64 [B]) encoded so that the signed 64-bit maximum over
 * shards is the full head's key: reduce with an int64 MAX all-reduce (8 bytes
 * per row), then decode with fs_keys_to_tokens.  The result is bitwise the
 * single-GPU fs_sample_ex result.  mask_bits, if given, covers the full
 * vocabulary, uint32 [B][ceil(V_total/32)].  Other arguments as fs_sample_ex;
 * a row with no allowed token in the shard gets the smallest key. */
fs_status fs_sample_shard_keys(const void *H, const void *W_shard, int B, int d,
                               int V_shard, int vocab_offset, int V_total,
                               float temperature, uint64_t seed,
                               const uint64_t *row_seeds, uint32_t step,
                               const uint32_t *mask_bits, int64_t *out_keys,
                               void *workspace, size_t workspace_bytes,
                               fs_stream_t stream);

/* Decodes reduced keys (device int64 [B], from fs_sample_shard_keys and a
 * MAX reduction) into tokens out_idx (device int32 [B]); -1 where no shard
 * had an allowed token. */
fs_status fs_keys_to_tokens(const int64_t *keys, int B, int32_t *out_idx,
                            fs_stream_t stream);

/* ---- Tensor-parallel vocabulary sampling with the exchange fused into the
 * kernel (readus.org page, "distributed FlashSampling": every GPU is one
 * group and sends only its winner's index and score; abstract: the argmax
 * decomposes over any partition).  Instead of an all-reduce after the
 * kernel, the last CTA of each rank's kernel writes its rows' packed
 * (score, token) maxima straight into every rank's exchange area over
 * NVLink (atomic max on peer memory), counts itself in every area, and the
 * arrival that completes an area decodes it; no kernel waits for another.
 * The stream that needs the tokens then waits on the area's flag.
 *
 * Protocol for a group of `world` ranks (one process per GPU):
 *   1. each rank: fs_tp_area_create(&mine); fs_ipc_handle(mine, h) and
 *      exchange the handles (e.g. an all-gather); fs_ipc_open on every
 *      peer's handle; areas[r] = rank r's area as mapped in this process
 *      (areas[own rank] = mine).  Every rank uses the same order.
 *   2. call number seq = 0, 1, 2, ... (the same on every rank):
 *      fs_sample_tp(..., areas, world, seq, ...) then
 *      fs_tp_wait(mine, B, seq, out_idx, timeout_us, stream) on the same
 *      stream; out_idx holds the tokens once the stream gets there.
 *   3. at the end: fs_ipc_close on the peers' areas, fs_tp_area_destroy.
 * A rank must not issue call seq + 1 on a stream that has not passed its
 * fs_tp_wait of call seq (the alternate halves of the area rely on it).
 * If any rank's kernel records a device error, it still completes the
 * exchange; every rank then gets -1 for every row of that call and
 * fs_tp_failed reports the call.  If a peer never completes a call (its
 * process died, say), this rank's fs_tp_wait gives up after its time limit,
 * with the same -1 tokens and fs_tp_failed report; the areas are then in an
 * unknown state and must be recreated on every rank before further calls.
 * Sequence numbers wrap after 2^32 calls. */
#define FS_IPC_HANDLE_BYTES 64

/* Bytes of one exchange area (fixed; up to 256 rows per call). */
size_t fs_tp_area_bytes(void);

/* Allocates a zeroed exchange area on the current device (cudaMalloc, so
 * that it can be shared by IPC), or frees one. */
fs_status fs_tp_area_create(void **area);
fs_status fs_tp_area_destroy(void *area);

/* CUDA IPC for exchange areas: the FS_IPC_HANDLE_BYTES-byte handle of an
 * area created here, and opening (with peer access enabled) or closing a
 * peer's area in this process. */
fs_status fs_ipc_handle(const void *area, void *handle);
fs_status fs_ipc_open(const void *handle, void **area);
fs_status fs_ipc_close(void *area);

/* One rank's part of tensor-parallel sampling: samples the shard as
 * fs_sample_shard_keys does (same arguments; B <= 256, else
 * FS_ERR_UNSUPPORTED) and exchanges the result through `areas` (host array of
 * `world` <= 16 device pointers, each 256-byte aligned).  Asynchronous on
 * `stream`; follow it with fs_tp_wait.  The tokens equal single-GPU
 * fs_sample_ex on the full head bit for bit. */
fs_status fs_sample_tp(const void *H, const void *W_shard, int B, int d,
                       int V_shard, int vocab_offset, int V_total,
                       float temperature, uint64_t seed,
                       const uint64_t *row_seeds, uint32_t step,
                       const uint32_t *mask_bits, void *const *areas, int world,
                       uint32_t seq, void *workspace, size_t workspace_bytes,
                       fs_stream_t stream);

/* Enqueues on `stream` one small kernel that waits until call `seq` has
 * been decoded into this rank's area `area` (the flag the completing rank
 * stores with release semantics at system scope), for at most timeout_us
 * microseconds (1 .. 60,000,000, else FS_ERR_INVALID_ARG), then copies the
 * call's B <= 256 tokens to out_idx (device int32 [B]).  If the limit
 * passes first, every token is -1 and fs_tp_failed reports seq. */
fs_status fs_tp_wait(const void *area, int B, uint32_t seq, int32_t *out_idx,
                     uint32_t timeout_us, fs_stream_t stream);

/* Synchronous: seq + 1 of the last call decoded with a device error in
 * `area`, or whose fs_tp_wait on `area` ran out of time (0: none). */
fs_status fs_tp_failed(const void *area, uint32_t *failed);

/* Top-k sampling (readus.org page, "Top-K and masking": a fast prefilter
 * isolates the candidates, then exact Gumbel-max runs on that subset).  The
 * candidates of row b are its K allowed tokens with the largest logits l
 * (ties toward the smaller index; every allowed token if there are fewer),
 * and the token is the argmax over them of x + g with the same noise as
 * fs_sample_ex, so K >= V gives the fs_sample_ex token.  The matmul writes
 * fp32 logits to `logits` (device [B][V], caller-owned, as in
 * fs_sample_unfused); then two launches: every row is split over several
 * blocks, each of which narrows its slice to a candidate list by radix
 * histograms over the order-preserving bits (the lists together hold the
 * row's top K), and one block per row selects the exact top K from the
 * lists and samples.  The lists live in a library-owned device buffer
 * (allocated on first use and grown as needed: 8 x rows x P x
 * min(max(K, 2048), V / P) bytes for P blocks per row, 4 MB at 64 rows and
 * K <= 2048, at most about 8 x rows x V bytes), so top-k
 * calls on one device must not overlap on the GPU (order them on one
 * stream).  K >= 1; other arguments as fs_sample_ex. */
fs_status fs_sample_topk(const void *H, const void *W, int B, int d, int V,
                         int K, float temperature, uint64_t seed,
                         const uint64_t *row_seeds, uint32_t step,
                         const uint32_t *mask_bits, int32_t *out_idx,
                         float *logits, void *workspace, size_t workspace_bytes,
                         fs_stream_t stream);

/* End-to-end call with HOST buffers: H_host (bf16 [B, d]) and out_idx_host
 * (int32 [B]) are host pointers (page-locked for the copies to be
 * asynchronous); W and row_seeds/mask_bits stay device pointers.  Enqueues
 * the host-to-device copy of H into one of two library-owned device buffers,
 * used by alternate calls, on a library stream (after the kernel of the call
 * two back, which read that buffer; so the copy overlaps the previous
 * call's kernel), the fused sample on `stream` (it starts streaming W at
 * once and waits on the device, with the usual one-second limit, for the
 * copy of H to land), and the tokens: written by the kernel straight into
 * out_idx_host when it is page-locked, else copied from a device buffer on
 * `stream`; the tokens are valid once `stream` is synchronised.  H_host must
 * stay unchanged until then.  Without stream memory operations on the
 * device, the copy of H runs on `stream` before the sample. */
fs_status fs_sample_host(const void *H_host, const void *W, int B, int d,
                         int V, float temperature, uint64_t seed,
                         const uint64_t *row_seeds, uint32_t step,
                         const uint32_t *mask_bits, int32_t *out_idx_host,
                         fs_stream_t stream);

/* Allocation-free flat sampling: the same computation and arguments as
 * fs_sample_ex without a workspace.  It exists for callers that must not
 * call cudaMalloc: a serving engine or framework that owns all device memory
 * through its own pool and hands a plug-in only its inputs and outputs, or a
 * decode loop that cannot afford an allocation's latency and device-wide
 * synchronisation.  The other entry points either allocate a workspace on
 * their first call or need one from the caller; this one keeps its scratch
 * (status word, ticket counter, one packed key per row: 2,304 bytes) in a
 * fixed array inside the library's device memory, which every GPU that
 * loads the library holds until the process exits.  The paper has no
 * counterpart for this entry point.
 * Limit: B <= 256 rows per call; a larger B returns FS_ERR_UNSUPPORTED
 * (split the batch into several calls).  The first call on each device
 * looks up the array's device address and may load the library's device
 * code; make that first call before any stream capture.  Each call clears
 * the array's ticket and keys on `stream` before using them, and every call
 * on a device shares the same array: calls that overlap on the GPU
 * (different streams or threads) race, so the caller must order them.
 * Device-side errors: a kernel that gave up on a bounded wait records
 * FS_ERR_DEVICE_TIMEOUT in the array's own status word (not in any
 * workspace; fs_device_status does not see it) and leaves out_idx
 * unwritten; the word keeps it across later calls until fs_noalloc_status
 * reads and clears it. */
fs_status fs_sample_noalloc(const void *H, const void *W, int B, int d, int V,
                            float temperature, uint64_t seed,
                            const uint64_t *row_seeds, uint32_t step,
                            const uint32_t *mask_bits, int32_t *out_idx,
                            fs_stream_t stream);

/* Reads (synchronously, after `stream` drains) and clears the status word of
 * fs_sample_noalloc's fixed array on the current device: FS_OK, or
 * FS_ERR_DEVICE_TIMEOUT when a call since the last read gave up on a bounded
 * wait (its tokens were not written), or in the debug build
 * FS_ERR_DEVICE_BOUNDS when a bounds check failed; FS_OK too before the
 * first call.
 * Allocates nothing; like fs_sample_noalloc, it must not overlap such a call
 * on the GPU.  The paper has no counterpart for this entry point. */
fs_status fs_noalloc_status(fs_stream_t stream);

/* Bytes of caller workspace needed by the calls above for these sizes on the
 * current device (G = 0 or 1 for flat sampling).  Returns 0 on invalid sizes. */
size_t fs_workspace_bytes(int B, int V, int G);

/* Workspace bytes of fs_sample_multi on the current device (0 on invalid
 * sizes). */
size_t fs_workspace_bytes_multi(int B, int V, int num_samples);

/* Workspace bytes of fs_summarize_group for a group of V_g rows. */
size_t fs_workspace_bytes_summary(int B, int V_g);

/* Reads (synchronously, after the stream drains) and clears the device-side
 * status word of a workspace (NULL = the library-owned one on the current
 * device).  Returns FS_OK, FS_ERR_DEVICE_TIMEOUT, or (debug build only)
 * FS_ERR_DEVICE_BOUNDS; after either error the workspace is zero-filled again
 * so it can be reused.  fs_sample_noalloc
 * keeps its status in its own array: read it with fs_noalloc_status. */
fs_status fs_device_status(void *workspace, size_t workspace_bytes,
                           fs_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char *fs_status_string(fs_status status);

/* ---- Test entry points: the device noise primitives the kernels use ---- */

/* out[i][0..3] = Philox4x32-10(counter = ctr[i][0..3], key = key[i][0..1]),
 * n >= 0 counters; all pointers device uint32 arrays. */
fs_status fs_philox4x32_10(const uint32_t *ctr, const uint32_t *key,
                           uint32_t *out, int64_t n, fs_stream_t stream);

/* g[i] = fp32 Gumbel transform of the noise word r[i] (the same device
 * function the sampling kernels use); device arrays of n elements. */
fs_status fs_gumbel(const uint32_t *r, float *g, int64_t n,
                    fs_stream_t stream);

/* Failure-detection test switch: while on (1), every fused-kernel launch's
 * load-issuing warp issues nothing, so the kernel's bounded waits run out
 * after about one second and it records FS_ERR_DEVICE_TIMEOUT, as in
 * fs_test_stalled_sample; for exercising error paths of other entry points
 * (fs_sample_tp marks the exchanged call as failed).  Off (0) by default;
 * process-wide. */
fs_status fs_test_stall_loads(int on);

/* Failure-detection test: launches the flat kernel on these arguments with
 * its load-issuing warp told to issue nothing, so the MMA warp's wait for
 * data runs out after about one second; every CTA then records
 * FS_ERR_DEVICE_TIMEOUT in the workspace, drains, frees its tensor memory and
 * exits, leaving the context usable.  fs_device_status() on the same
 * workspace afterwards returns FS_ERR_DEVICE_TIMEOUT (and re-zeroes it).
 * out_idx is left unwritten.  Same argument rules as fs_sample_ex. */
fs_status fs_test_stalled_sample(const void *H, const void *W, int B, int d,
                                 int V, int32_t *out_idx, void *workspace,
                                 size_t workspace_bytes, fs_stream_t stream);

/* Host-side fault injection for failure-detection tests (nothing is done to
 * the GPU).  kind 1 ("alloc"): every device allocation the library would
 * make fails; kind 2 ("launch"): every call that would enqueue work on a
 * stream fails; either way the call returns FS_ERR_CUDA before it touches
 * the GPU, and the library stays usable once the kind is back to 0 (none).
 * The initial kind comes from the environment variable FS_FAULT ("alloc" or
 * "launch"; anything else is none), read at the first call.  kind -1 leaves
 * the setting as it is; *previous (if not NULL) receives the kind in force
 * before the call.  Process-wide.  FS_ERR_INVALID_ARG for kind < -1 or > 2. */
fs_status fs_test_inject_fault(int kind, int *previous);

/* ---- Kernel choice ---- */

/* Whether flat-mode calls (fs_sample, fs_sample_ex, fs_sample_host,
 * fs_sample_noalloc, fs_sample_multi, fs_sample_shard_keys) and grouped calls
 * (fs_sample_grouped, fs_summarize_group) run the fused kernel on CTA pairs:
 * clusters of two CTAs on two SMs that share one M = 256 tensor-core MMA
 * (tcgen05 cta_group::2), each SM staging 128 rows of W and half of the batch
 * rows of H per pipeline stage.  On pairs with a 256-row batch tile, a
 * partial tile of at most 240 vocabulary rows is multiplied transposed (the
 * batch rows as the MMA's M operand), so that it costs its own width of MMA
 * work rather than a whole tile's.  This is a B200 design choice, not part of
 * the method: the results are the same either way (tokens bit for bit).
 * policy: -1 automatic (the default: pairs for launches whose batch tile,
 * the row count rounded up to a multiple of 16, is 112 or more, i.e. from
 * 97 rows per launch; fs_plan_batch reports the choice), 0 never, 1 always.
 * Process-wide; applies to calls made after it returns.  FS_ERR_INVALID_ARG
 * for any other value.  When the device
 * cannot co-schedule a pair, the single-CTA kernel runs.  The unfused
 * measurement path (fs_sample_unfused, fs_sample_topk) always runs on single
 * CTAs. */
fs_status fs_set_cta_pairs(int policy);

/* Whether the fused kernel is launched as a programmatic dependent of the
 * kernel ahead of it in the stream (CUDA programmatic dependent launch):
 * on (1, the default), for launches whose batch tile is at most 128 rows
 * (where W streaming sets the time), back-to-back calls overlap, the next
 * kernel's CTAs starting on the SMs the previous one has left and streaming
 * W at once, while its loads of H and every access to the workspace wait
 * until the previous kernel has completed (H may be that kernel's output);
 * larger tiles, tensor-bound, run in plain order.  Off (0): plain stream
 * order for every launch.  The tokens are the same either way (bit for bit).  A
 * B200 scheduling choice, not part of the method.  Process-wide; applies to
 * calls made after it returns.  FS_ERR_INVALID_ARG for any other value. */
fs_status fs_set_programmatic_launch(int on);

/* The execution-path choices in force: *cta_pairs and *partial_merge (-1
 * automatic, 0 never, 1 always, as set by fs_set_cta_pairs and
 * fs_set_partial_merge), *programmatic (fs_set_programmatic_launch),
 * *unfused (1 when flat single-sample calls run the unfused two-kernel mode)
 * and *two_kernel_reduce (1 when flat calls leave the per-row maxima to a
 * second, decoding kernel instead of the fused kernel's last CTA; the fused
 * tensor-parallel exchange always uses the last CTA).  The initial choices
 * come from the environment variable FS_FORCE_PATH, read once at the first
 * call that uses them: a comma-separated list of "unfused" or "fused"
 * (fs_sample and fs_sample_ex run the measurement mode of fs_sample_unfused,
 * fp32 logits through HBM in a library-owned buffer, or the fused kernel),
 * "twokernel" or "lastcta", "pairs" or "single", "merge" or "nomerge",
 * "plain" or "programmatic"; unknown words are ignored, and the fs_set_*
 * calls override it afterwards.  Every choice gives the same tokens.  For A/B
 * runs without code changes.  Host-only; NULL pointers are skipped. */
fs_status fs_get_policies(int *cta_pairs, int *partial_merge, int *programmatic,
                          int *unfused, int *two_kernel_reduce);

/* Kernel choice for single-CTA launches of up to 64 batch rows: a CTA whose
 * vocabulary range starts with an 8-row partial tile can either run it as a
 * tile of its own (which streams all of H again for 8 rows of W) or multiply
 * it in the same pipeline stages as its first whole tile, sharing the H
 * loads (a 1 KB slot per stage for its rows, a second MMA into its own
 * accumulator).  The results are the same either way (tokens bit for bit);
 * the merged variant pays where many CTAs have such a tile (the Qwen3 heads,
 * 48 of 148) and costs a little ring space elsewhere.  policy: -1 automatic
 * (the default: merge when at least one CTA in ten has one), 0 never,
 * 1 always.  Process-wide; applies to calls made after it returns.
 * FS_ERR_INVALID_ARG for any other value. */
fs_status fs_set_partial_merge(int policy);

/* ---- Host-only schedule query (no GPU needed) ---- */

/* The vocabulary schedule of the fused kernel for V tokens, G groups
 * (0 or 1: flat) on `num_sms` SMs (the number of persistent CTAs it
 * launches is returned in *num_ctas_out if not NULL).  Writes up to
 * max_tiles rows of int32 [5] = (tile start, first valid token, end of valid
 * tokens, partial slot, last-tile-of-segment flag) for CTA `cta` and returns
 * the count in *ntiles.  Tiles are 128 tokens; a CTA's range is a multiple
 * of 8 tokens (except at V); a tile never crosses a group boundary.  A launch
 * on CTA pairs splits the vocabulary over its pair units in the same way
 * (the query with num_sms = the number of units, 74 on a 148-SM device) and
 * walks each segment in 256-token tiles, its partial tile first; with a
 * 256-row batch tile a partial tile of at most 240 tokens is multiplied
 * transposed (see fs_set_cta_pairs).  (With
 * merged partial tiles, fs_set_partial_merge, the kernel multiplies an 8-row
 * partial tile in the same pipeline stages as the tile after it; the tiles
 * and slots listed here stay the same.) */
fs_status fs_plan_tiles(int V, int G, int num_sms, int cta, int32_t *tiles,
                        int max_tiles, int *ntiles, int *num_ctas_out);

/* The same schedule as the kernel variant with merged partial tiles runs it
 * (single-CTA launches of at most 64 rows; fs_set_partial_merge): rows of
 * int32 [8] = the five columns above, then (partial start, first valid
 * token, end of valid tokens) of the 8-row partial tile multiplied in the
 * same stages as this tile, or (-1, 0, 0) for none.  Expanding every merged
 * partial into a tile of its own, just before its tile and with the same
 * slot, gives fs_plan_tiles' list.  *merges (if not NULL) = 1 when the
 * automatic choice runs this variant for the split (at least one CTA in ten
 * starts a segment with an 8-row partial tile), else 0. */
fs_status fs_plan_tiles_merged(int V, int G, int num_sms, int cta, int32_t *tiles,
                               int max_tiles, int *ntiles, int *merges);

/* How a call of B rows is launched: *launches = fused-kernel launches (one
 * per 256 rows), *batch_tile = the first launch's batch tile (MMA N: the
 * row count rounded up to a multiple of 16, at most 256), *cta_pairs = 1 when
 * the current fs_set_cta_pairs policy runs it on CTA pairs (on a device
 * that can co-schedule them), else 0.  kind: 0 flat (fs_sample and the
 * other flat-mode calls), 1 grouped, 2 unfused / top-k (logits mode, single
 * CTAs).  Output pointers other than `launches` may be NULL.  Host-only. */
fs_status fs_plan_batch(int B, int kind, int *launches, int *batch_tile, int *cta_pairs);

/* The CTAs whose vocabulary range meets group g (0 <= g < G), as the grouped
 * merge kernel enumerates them: [*first, *last].  Host-only. */
fs_status fs_plan_group_ctas(int V, int G, int num_sms, int g, int *first,
                             int *last);

#ifdef __cplusplus
}
#endif

#endif /* FMMS_H_ */
