/*
 * aoh.h -- C ABI of the token-sparse decode library (libaoh.so).
 *
 * One decode step of token-sparse attention over a long KV cache, on one
 * sm_100a GPU:
 *   1. importance scores from the dominant RoPE frequency chunks of each KV
 *      head (FASA: Frequency-aware Sparse Attention, section 2.B.1, Token
 *      Importance Predictor; chunks as defined in section 2.A),
 *   2. a per-(sequence, KV head) top-N_fac selection of those scores
 *      (same section),
 *   3. exact full-dimension softmax attention over only the selected tokens
 *      at their original positions (section 2.B.2, Focused Attention
 *      Computation; the whole cache stays on the GPU and only part of K is
 *      read, as in the FASA-C variant of section 2.C).
 * Around it: the retrieval / streaming head-role split of the AoH summary
 * (Resumen Tecnico: Autonomia de Cabezales, Metodologia section 4:
 * retrieval heads attend to the whole cache, streaming heads to a sink plus
 * a recent window), and the shared index of the CLSA article (El
 * enrutamiento compartido entre capas..., "Como funciona CLSA": one top-k,
 * computed once, reused by every cross-decoder layer over a shared cache).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every buffer is owned by the caller.  Pointers marked "device" must be
 *   device memory of the current CUDA device; "host" pointers are read
 *   during the call only.  The library allocates no memory.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *   asynchronous: they validate their arguments on the host, enqueue kernels
 *   on `stream` and return.  No call synchronises, except aoh_device_check.
 * - Errors come back as aoh_status; nothing is thrown across the ABI.
 *   Argument errors are found on the host before anything is launched and
 *   leave every output untouched.  A failed launch returns AOH_ERR_CUDA.
 *   Conditions only the device can see (a stored position outside its
 *   sequence, a per-sequence N_fac above the capacity, a chunk id outside
 *   [0, d/2)) are recorded in a per-device error word, the offending access
 *   is skipped, and aoh_device_check() reports them.
 * - Tensors are bf16 (raw 16-bit storage) unless stated otherwise; outputs
 *   are fp32.  Keys and queries are already rotated by RoPE at their
 *   absolute positions (keys of sequence b at 0..L_b-1, its query at L_b);
 *   nothing here rotates, so "original positions" hold by construction.
 * - GQA: q head h reads KV head g = h / G with G = n_q_heads / n_kv_heads
 *   (contiguous groups).
 */
#ifndef AOH_H
#define AOH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AOH_OK = 0,
  AOH_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent shapes          */
  AOH_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim not 64/128) */
  AOH_ERR_ALIGNMENT = 3,     /* a pointer or stride breaks the 16-byte row rule      */
  AOH_ERR_WORKSPACE = 4,     /* workspace NULL, too small or not 256-byte aligned    */
  AOH_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed                 */
  AOH_ERR_DEVICE_CHECK = 6   /* a device-side check fired (see aoh_device_check)     */
} aoh_status;

/* Head roles, one per KV head (AoH summary, Metodologia section 4). */
enum {
  AOH_ROLE_SPARSE = 0, /* importance score -> top-N_fac -> focused attention      */
  AOH_ROLE_DENSE = 1,  /* retrieval head: attention over every cached token        */
  AOH_ROLE_STREAM = 2  /* streaming head: sink tokens plus the recent window only  */
};

/*
 * The KV cache of one decode step (ragged batch).
 *
 * Element i of KV head h of global token t is at
 *   k[t * stride_tok + h * stride_head + i]   (same for v),
 * where sequence b owns global tokens [offsets[b], offsets[b+1]) and its
 * local position p is global token offsets[b] + p.  head_dim elements of a
 * row are contiguous.  k and v must be 16-byte aligned and both strides
 * multiples of 8 elements (every row starts on a 16-byte boundary).
 *
 * k_dom (optional) is a packed copy of the dominant columns of K, laid out
 * [head slots][total_tokens][k_dom_cols]: in row (slot of h, t), column
 * j < n_dom holds K dim I_dom[h][j], column n_dom + j holds dim I_dom[h][j] +
 * d/2, the rest (up to k_dom_cols, a multiple of 8) are zero.
 * aoh_pack_dominant writes it, aoh_kv_append extends it.  With it the
 * importance scan reads 4 * n_dom bytes per token and head instead of the
 * sectors of K that the chunks touch.
 *
 * Lengths and capacity (ABI 2).  With lengths == NULL sequence b fills its
 * region [offsets[b], offsets[b+1]): L_b = offsets[b+1] - offsets[b].  With
 * lengths, sequence b holds positions 0 .. lengths[b] - 1 and its region is
 * its capacity; tokens of the region past the length are never read.
 *
 * Head slots (ABI 2).  KV head g's rows are stored in head slot s =
 * head_slot[g] (identity when head_slot is NULL): element i of position p is at
 * k[t * stride_tok + s * stride_head + i] with t the position's token.  A
 * cache need not store every head: AOH_NO_SLOT marks a head it does not store,
 * and every call on that cache skips such heads.  So the retrieval heads of the
 * AoH split can live in one cache (the whole history) and the streaming heads in
 * a ring (below), each sized for the heads it holds.
 *
 * Layouts.  ring_sink = ring_window = 0: the linear layout, position p is
 * token offsets[b] + p (lengths[b] <= offsets[b+1] - offsets[b], else device
 * check 4 and the length is clamped).  Otherwise the ring layout of a streaming
 * head's cache (AoH summary, Metodologia section 4: a fixed sink plus a recent
 * window): the region holds ring_sink + ring_window slots, position p < sink
 * is slot p and a later position is slot sink + (p - sink) mod window, so
 * after L tokens the ring holds exactly positions [0, min(sink, L)) and
 * [max(sink, L - window), L).  Only aoh_stream_decode (STREAM heads) and
 * aoh_kv_append use a ring; the other calls refuse it.
 */
typedef struct aoh_kv_cache {
  const void* k;               /* device, bf16                                         */
  const void* v;               /* device, bf16                                         */
  const int32_t* offsets;      /* device int32 [batch + 1], non-decreasing, offsets[0]=0 */
  int32_t batch;               /* number of sequences B (0 is a no-op)                 */
  int32_t n_kv_heads;          /* Hkv, 1..128                                          */
  int32_t head_dim;            /* d: 64 or 128                                         */
  int32_t max_len;             /* host copy of max_b L_b (an upper bound is fine)       */
  int64_t total_tokens;        /* host copy of offsets[batch], < 2^31                  */
  int64_t stride_tok;          /* elements between tokens t and t+1 of one head        */
  int64_t stride_head;         /* elements between heads h and h+1 of one token        */
  const void* k_dom;           /* device bf16 [slots][total_tokens][k_dom_cols], or NULL */
  int32_t k_dom_cols;          /* row length of k_dom in elements (0 when k_dom NULL)  */
  /* ABI 2 (zero-filled: the ABI 1 meaning) */
  const int32_t* lengths;      /* device int32 [batch] or NULL: positions held per sequence */
  const uint8_t* head_slot;    /* host uint8 [n_kv_heads] or NULL (identity); read per call */
  int32_t ring_sink;           /* ring layout: sink slots (0 and 0: linear layout)      */
  int32_t ring_window;         /* ring layout: window slots                            */
} aoh_kv_cache;

#define AOH_NO_SLOT 255        /* head_slot entry of a head the cache does not store    */

/* Human-readable name of a status code (static string). */
const char* aoh_status_string(aoh_status s);

/* Library ABI version: 2 (1 plus lengths, head slots and rings in aoh_kv_cache,
 * and aoh_kv_append). */
int32_t aoh_version(void);

/* The cudaError_t code behind the last AOH_ERR_CUDA returned on the calling
 * host thread (0 if none); cudaGetErrorString() names it. */
int32_t aoh_last_cuda_error(void);

/* Kernels the library launches, one counter each (see aoh_launch_counts). */
typedef enum {
  AOH_KERNEL_TIP_SCORE = 0,     /* stand-alone importance scan                       */
  AOH_KERNEL_SELECT_HIST = 1,   /* select: first-digit histograms of given scores    */
  AOH_KERNEL_SPARSE_ROW = 2,    /* fused row kernel                                  */
  AOH_KERNEL_FLASH_GATHER = 3,  /* split-K gather / window attention                 */
  AOH_KERNEL_PACK_DOMINANT = 4, /* dominant-column packing of K                      */
  AOH_KERNEL_KV_APPEND = 5,     /* rotation and append of a decoded token            */
  AOH_KERNEL_GRAM = 6,          /* head classifier: W W^T of every head (tensor cores) */
  AOH_KERNEL_GRAM_REDUCE = 7,   /* head classifier: fp64 sum of the split partials   */
  AOH_KERNEL_SPECTRUM = 8,      /* head classifier: Cholesky, congruence, Jacobi, ER */
  AOH_KERNEL_GROUP_ROLES = 9,   /* head classifier: group means and roles            */
  AOH_KERNEL_OFFLOAD_STAGE = 10,  /* host offload: selected rows across the host link */
  AOH_KERNEL_OFFLOAD_SPLIT = 11,  /* host offload: a device cache split to host parts */
  AOH_KERNEL_SELECT_CHUNK = 12, /* select: threshold bin, counts above it, candidates */
  AOH_KERNEL_SELECT_WRITE = 13, /* select: ordered write of the chosen positions     */
  AOH_KERNEL_SELECT_CLUSTER = 14, /* select: one cluster per row, keys on chip      */
  AOH_KERNEL_SELECT_RESOLVE = 15, /* select: exact threshold and chunk offsets per row */
  AOH_KERNEL_FLASH_MERGE = 16,  /* split-K combine of rows with many splits           */
  AOH_KERNEL_KINDS = 17
} aoh_kernel_kind;

/*
 * aoh_launch_counts -- kernel launches this process has made through the
 * library, by kernel.  Host-side counters, incremented at every launch the
 * runtime accepted (a launch captured into a CUDA graph counts once, at
 * capture; graph replays do not count).  Writes min(n, AOH_KERNEL_KINDS)
 * host int64 to `counts` (may be NULL when n is 0); returns AOH_KERNEL_KINDS.
 * Differences of two readings around a call give that call's launches.
 */
int32_t aoh_launch_counts(int64_t* counts, int32_t n);

/*
 * aoh_record_launch_events -- diagnostic timing of the kernels inside a call.
 * While armed (events not NULL), the next launch records events[0] on its
 * stream just before it, and launch i (1-based) records events[i] just after
 * it and writes its aoh_kernel_kind to kinds[i - 1], for i < n; later
 * launches record nothing.  cudaEventElapsedTime(events[i - 1], events[i])
 * is then the device time of launch i.  `events`: host array of n
 * cudaEvent_t created by the caller; `kinds`: host int32[n - 1] or NULL.
 * Both must stay valid until the call is repeated with events = NULL, which
 * disarms it.  Process-wide and not thread-safe: for measurement only.
 */
void aoh_record_launch_events(void** events, int32_t* kinds, int32_t n);

/*
 * aoh_device_check -- synchronise `stream`, then read and clear this
 * device's error word.  Returns AOH_OK, AOH_ERR_DEVICE_CHECK (and, if
 * `detail` is not NULL, writes 4 host int32: check id, then three values of
 * the first failing access), or AOH_ERR_CUDA.  Check ids: 1 a position
 * outside [0, L_b) or offsets past the cache, 2 a count or per-sequence
 * N_fac above the capacity, 3 a chunk id outside [0, d/2), 4 a sequence
 * length or appended position past its region's capacity (or a ring region
 * smaller than its slots), 5 a key Gram matrix without a Cholesky factor
 * (aoh_head_classify: a key block without full row rank).
 */
aoh_status aoh_device_check(void* stream, int32_t* detail);

/*
 * aoh_pack_dominant -- write the packed dominant-column copy of K
 * (layout in aoh_kv_cache above).  A cache-maintenance step: run it when
 * tokens are appended, not per decode step.  FASA section 2.C (FASA-M keeps
 * only the dominant parts of K on the GPU; this is that layout kept beside
 * the full cache).
 *   idom     device int32 [n_kv_heads][n_dom], chunk ids in [0, d/2)
 *   n_dom    1 .. d/2, and 2*n_dom <= k_dom_cols
 *   k_dom    device bf16 [n_kv_heads][kv->total_tokens][k_dom_cols], 16-B aligned
 *   k_dom_cols  multiple of 8
 * kv->k_dom is ignored here.
 */
aoh_status aoh_pack_dominant(const aoh_kv_cache* kv, const int32_t* idom, int32_t n_dom,
                             void* k_dom, int32_t k_dom_cols, void* stream);

/*
 * aoh_tip_score -- importance of every cached token (FASA section 2.B.1,
 * with GQA aggregation by summing over the group, AoH section 4):
 *   scores[g][t] = sum over q heads h of group g, over c in I_dom[g], of
 *                  q_h[c] * k_t[c] + q_h[c + d/2] * k_t[c + d/2]
 * computed as one fp32 dot of the fp32 group sum of q with the dominant
 * columns of k_t.  No 1/sqrt(d) scale.
 *   q        device bf16 [B][n_q_heads][d], contiguous
 *   idom     device int32 [Hkv][n_dom], chunk ids in [0, d/2).  With every
 *            chunk listed (n_dom = d/2) the score is the full q.k of the
 *            group sum: the shared indexer's score.
 *   scores   device fp32 [Hkv][kv->total_tokens]; entry (g, offsets[b] + p)
 *            is token p of sequence b.
 * If kv->k_dom is set it must have been packed with this idom / n_dom and
 * the scan reads it; otherwise K is read in place.
 */
aoh_status aoh_tip_score(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv,
                         const int32_t* idom, int32_t n_dom, float* scores, void* stream);

/*
 * aoh_topk_select -- per (sequence b, KV head g): the n = min(N_fac_b, L_b)
 * positions with the largest scores (FASA section 2.B.1; the shared index's
 * single top-k).  Equal scores: the lower position wins; -0 equals +0.
 * Output positions are ascending.
 *   scores          device fp32 [Hkv][total_tokens] (layout of aoh_tip_score);
 *                   finite values
 *   n_fac           N_fac for every sequence when n_fac_per_seq is NULL
 *   n_fac_per_seq   device int32 [B] or NULL
 *   n_fac_cap       capacity per row; n_fac (or every n_fac_per_seq entry) <= cap
 *   idx             device int32 [B][Hkv][n_fac_cap]; entries >= n are set to -1
 *   count           device int32 [B][Hkv]: n
 *   workspace       device, 256-byte aligned, >= aoh_topk_select_workspace_size
 *                   bytes, zero-filled once before its first use (every call
 *                   leaves its counters at zero again)
 * Rows up to 4 M positions (AOH_ERR_UNSUPPORTED beyond).  Deterministic: the
 * same input gives the same bits.  Mechanism, on order-preserving uint32 keys,
 * in one of three forms:
 *  - rows of at most 128 K positions whose clusters fit one wave: one launch,
 *    one thread-block cluster per row with the row's keys in registers (MSB
 *    radix select with 11-, 11- and 10-bit digits, histograms summed across
 *    the cluster through distributed shared memory, picks written in order);
 *  - else, fewer rows than SMs of at most 256 K positions that fit one wave of
 *    the fused row kernel's clusters: that kernel in its select-only mode (keys
 *    in shared memory, 8-bit digits), one launch;
 *  - else four launches: a histogram of the top 11 bits; chunks of 4096 keys
 *    in parallel (keys above the threshold bin counted, keys in it collected);
 *    one CTA per row resolving the exact threshold and every chunk's offset;
 *    every chunk's picks written in order.
 */
aoh_status aoh_topk_select(const float* scores, const aoh_kv_cache* kv, int32_t n_fac,
                           const int32_t* n_fac_per_seq, int32_t n_fac_cap,
                           int32_t* idx, int32_t* count, void* workspace,
                           size_t workspace_bytes, void* stream);

size_t aoh_topk_select_workspace_size(const aoh_kv_cache* kv);

/*
 * aoh_sparse_decode -- the whole sparse step for the heads whose role is
 * AOH_ROLE_SPARSE: importance scores, top-N_fac, then exact attention of
 * every q head of the group over the selected tokens (FASA sections 2.B.1
 * and 2.B.2):
 *   out[b][h] = sum over selected t of softmax_t(scale * q_h . k_t) * v_t
 * in fp32 (online softmax, split over the selection, then combined).
 *   q, idom, n_dom, n_fac, n_fac_per_seq, n_fac_cap: as above
 *   roles      host uint8 [Hkv] or NULL (= every head SPARSE); only rows of
 *              SPARSE heads are computed and written
 *   scale      softmax scale, usually 1/sqrt(d)
 *   out        device fp32 [B][n_q_heads][d]
 *   idx_out, count_out   optional device outputs of the selection (layouts of
 *              aoh_topk_select, rows of non-SPARSE heads untouched), or NULL
 *   workspace  device, 256-byte aligned, >= aoh_sparse_decode_workspace_size
 *              bytes, zero-filled once before its first use (every call
 *              leaves its counters at zero again)
 * A sequence with L_b = 0 gives zero rows.
 */
aoh_status aoh_sparse_decode(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv,
                             const int32_t* idom, int32_t n_dom, int32_t n_fac,
                             const int32_t* n_fac_per_seq, int32_t n_fac_cap,
                             const uint8_t* roles, float scale, float* out,
                             int32_t* idx_out, int32_t* count_out,
                             void* workspace, size_t workspace_bytes, void* stream);

size_t aoh_sparse_decode_workspace_size(const aoh_kv_cache* kv, int32_t n_q_heads,
                                        int32_t n_fac_cap);

/*
 * aoh_stream_decode -- attention for the heads whose role is AOH_ROLE_DENSE
 * (every position [0, L_b)) or AOH_ROLE_STREAM (positions
 * [0, min(sink, L_b)) together with [max(0, L_b - window), L_b)); AoH
 * summary, Metodologia section 4.  Same arithmetic as aoh_sparse_decode.
 *   roles      host uint8 [Hkv] (required)
 *   sink, window >= 0
 *   out        device fp32 [B][n_q_heads][d]; only DENSE / STREAM rows written
 *   workspace  as for aoh_sparse_decode, >= aoh_stream_decode_workspace_size
 * Calling aoh_sparse_decode and aoh_stream_decode on the same `out` with the
 * same roles gives the full head-role-split decode step.
 */
aoh_status aoh_stream_decode(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv,
                             const uint8_t* roles, int32_t sink, int32_t window, float scale,
                             float* out, void* workspace, size_t workspace_bytes, void* stream);

size_t aoh_stream_decode_workspace_size(const aoh_kv_cache* kv, int32_t n_q_heads,
                                        const uint8_t* roles, int32_t sink, int32_t window);

/*
 * aoh_stream_decode_noalloc -- aoh_stream_decode without a caller workspace.  The
 * pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory: code that runs inside someone else's pre-reserved
 * memory pool or a plugin host that owns every device allocation, and
 * latency-critical paths where a cudaMalloc, with the device-wide
 * synchronisation it may imply, is not acceptable.
 *
 * The split-K scratch lives in a file-scope device array of 16 MiB that every
 * device which loads the library keeps until the process exits; the call
 * allocates nothing.  Arguments and results are those of aoh_stream_decode.
 *   - Returns AOH_ERR_WORKSPACE, without launching, when the step needs more
 *     than 16 MiB of scratch (aoh_stream_decode_workspace_size gives the need).
 *   - Every call looks the array's address up with the current device (a host
 *     query).  The first call on a device sets the array up: it zeroes it and
 *     synchronises the device, so make that first call before any stream
 *     capture.  A cudaDeviceReset destroys the array with its context; the next
 *     call finds the new address and sets the array up again (so, again, not
 *     during a capture).
 *   - Arguments are validated before the array is touched; a refused call
 *     leaves it as it was.  A kernel that was aborted (a lost context) can
 *     leave its split counters set; only a reset clears them.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; calls that can overlap on the GPU (different streams without
 *     ordering) race on it.  Serialise them on one stream.
 */
aoh_status aoh_stream_decode_noalloc(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv,
                                     const uint8_t* roles, int32_t sink, int32_t window,
                                     float scale, float* out, void* stream);

/*
 * aoh_decode_step -- the whole head-role-split step in one call: the SPARSE
 * heads as aoh_sparse_decode, the DENSE / STREAM heads as aoh_stream_decode,
 * on the same `out`.  When the fused row kernel holds every row in one wave
 * and no window head's list exceeds 4 * n_fac_cap positions, DENSE / STREAM
 * heads ride in the same launch as the SPARSE ones (their clusters attend over
 * their ranges without scan or select): one launch for the whole step.
 * Otherwise it runs the two calls in turn.  Arguments as for those two calls;
 * roles may be NULL (every head SPARSE); a ring cache takes window heads only.
 *   workspace  >= aoh_decode_step_workspace_size bytes, 256-byte aligned,
 *              zero-filled once before its first use
 */
aoh_status aoh_decode_step(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv,
                           const int32_t* idom, int32_t n_dom, int32_t n_fac,
                           const int32_t* n_fac_per_seq, int32_t n_fac_cap, const uint8_t* roles,
                           int32_t sink, int32_t window, float scale, float* out,
                           int32_t* idx_out, int32_t* count_out, void* workspace,
                           size_t workspace_bytes, void* stream);

size_t aoh_decode_step_workspace_size(const aoh_kv_cache* kv, int32_t n_q_heads, int32_t n_fac_cap,
                                      const uint8_t* roles, int32_t sink, int32_t window);

/*
 * aoh_shared_index_decode -- the cross-decoder layers of a shared-cache
 * stack reuse one index ("Como funciona CLSA"): for every layer l, every
 * q head h of group g and sequence b,
 *   out[l][b][h] = sum over t in idx[b][g][0 .. count[b][g]) of
 *                  softmax_t(scale * q_layers[l][b][h] . k_t) * v_t.
 * The index is read once per (b, g) and the K / V rows it names are read
 * once for all n_layers * G query rows.  Build the index with
 * aoh_tip_score (idom = every chunk 0..d/2-1) and aoh_topk_select.
 *   q_layers   device bf16 [n_layers][B][n_q_heads][d], contiguous
 *   n_layers * (n_q_heads / n_kv_heads) <= 32
 *   idx, count, n_fac_cap: layouts of aoh_topk_select; positions must lie in
 *              [0, L_b) (checked on the device)
 *   out        device fp32 [n_layers][B][n_q_heads][d]
 *   workspace  as above, >= aoh_shared_index_decode_workspace_size
 */
aoh_status aoh_shared_index_decode(const void* q_layers, int32_t n_layers, int32_t n_q_heads,
                                   const aoh_kv_cache* kv, const int32_t* idx,
                                   const int32_t* count, int32_t n_fac_cap, float scale,
                                   float* out, void* workspace, size_t workspace_bytes,
                                   void* stream);

size_t aoh_shared_index_decode_workspace_size(const aoh_kv_cache* kv, int32_t n_layers,
                                              int32_t n_q_heads, int32_t n_fac_cap);

/*
 * aoh_shared_index_step -- the whole shared-index stack step ("Como funciona
 * CLSA": the indexer scores the cache once, takes one top-k and every
 * cross-decoder layer attends over it).  Equivalent to aoh_tip_score (every
 * chunk, q_index) + aoh_topk_select (k = topk) + aoh_shared_index_decode.
 * When every (sequence, KV head) row fits one wave of thread-block clusters
 * the step is a single launch (scan, select, attention and combine per
 * cluster); otherwise it runs the scan over all SMs, the cluster select and
 * the split-K gather.
 *   q_index    device bf16 [B][n_q_heads][d]: the indexer layer's queries
 *   q_layers   device bf16 [n_layers][B][n_q_heads][d]
 *   n_layers * (n_q_heads / n_kv_heads) <= 32
 *   idx, count device outputs, layouts of aoh_topk_select with n_fac_cap = topk
 *   out        device fp32 [n_layers][B][n_q_heads][d]
 *   workspace  device, 256-byte aligned, zero-filled once before first use,
 *              >= aoh_shared_index_step_workspace_size bytes
 */
aoh_status aoh_shared_index_step(const void* q_index, const void* q_layers, int32_t n_layers,
                                 int32_t n_q_heads, const aoh_kv_cache* kv, int32_t topk,
                                 int32_t* idx, int32_t* count, float scale, float* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

size_t aoh_shared_index_step_workspace_size(const aoh_kv_cache* kv, int32_t n_layers,
                                            int32_t n_q_heads, int32_t topk);

/*
 * aoh_kv_append -- add the decoded token of every sequence to the caches.
 * The token's key and query are rotated by RoPE to its absolute position p
 * (FASA section 2.A: chunk c = dims (c, c + d/2) turned by p * theta^(-2c/d);
 * angles and rotation in double precision, stored as bf16 rounded to nearest,
 * ties to even); its key and value rows go to every cache that stores the
 * head: the linear cache for retrieval heads (the whole history) and the ring
 * for streaming heads (sink plus recent window), as the AoH summary's
 * Metodologia section 4 deploys them; the packed dominant row of each head the
 * linear cache stores is written when it has k_dom (FASA section 2.C).
 *   q_new      device bf16 [B][n_q_heads][d], before rotation, or NULL
 *   k_new, v_new  device bf16 [B][Hkv][d]: the key before rotation, the value
 *   theta      RoPE base (> 0)
 *   kv         the linear cache (ring_sink = ring_window = 0), or NULL
 *   ring       a ring-layout cache with the same batch / heads / head_dim, or
 *              NULL.  Every KV head must be stored by kv or ring (or both).
 *              The descriptors' own lengths fields are not used here.
 *   idom, n_dom  I_dom of every KV head, required when kv->k_dom is set
 *   lengths    device int32 [B]: p = lengths[b] is the new token's position;
 *              after the rows are written lengths[b] = p + 1
 *   q_out      device bf16 [B][n_q_heads][d]: q rotated to p (NULL iff q_new is)
 * A sequence whose linear region is full (p >= offsets[b+1] - offsets[b]), or
 * whose ring region has fewer than ring_sink + ring_window tokens, is left
 * unchanged (lengths included) and device check 4 is recorded.  Decoding after
 * the append attends over positions 0 .. p: the new token included.
 */
aoh_status aoh_kv_append(const void* q_new, int32_t n_q_heads, const void* k_new, const void* v_new,
                         double theta, const aoh_kv_cache* kv, const aoh_kv_cache* ring,
                         const int32_t* idom, int32_t n_dom, int32_t* lengths, void* q_out,
                         void* stream);

/*
 * aoh_head_classify -- the AoH offline head classifier on frozen projection
 * weights (AoH summary, Metodologia sections 1-4).  For q head h, whose keys
 * are KV head g = h / G, with W^h its d_head x d_model block of rows:
 *   M_h = W_K^g^T W_Q^h (section 1); its non-zero singular values are the
 *   square roots of the eigenvalues of C_h = (W_Q^h W_Q^h^T)(W_K^g W_K^g^T)
 *   (section 3); ER(h) = exp(-sum sigma_hat log sigma_hat) with sigma_hat =
 *   sigma / sum sigma over the values above 1e-12 of the largest (section 2);
 *   the group's ER is the mean over its q heads (GQA aggregation, section 4)
 *   and the n_retrieval lowest groups are retrieval heads (AOH_ROLE_DENSE),
 *   the rest streaming heads (AOH_ROLE_STREAM); equal ER: lower KV head first.
 * The Gram matrices run on tensor cores (bf16 products, fp32 sums of at most
 * 512 terms, summed over d_model in fp64); the spectrum is computed in fp64
 * (Cholesky of the key Gram B = L L^T, S = L^T A L whose eigenvalues are
 * those of C_h, cyclic Jacobi).  An offline step: run once per model.
 *   w_q        device bf16 [n_q_heads * head_dim][d_model], row-major (the
 *              q projection weight, one head's block of rows after another)
 *   w_k        device bf16 [n_kv_heads * head_dim][d_model], row-major
 *   d_model    multiple of 64, >= head_dim; head_dim 64 or 128
 *   n_retrieval  0 .. n_kv_heads
 *   er_heads   device float64 [n_q_heads]; er_groups device float64 [n_kv_heads]
 *   roles      device uint8 [n_kv_heads]: AOH_ROLE_DENSE or AOH_ROLE_STREAM
 *   workspace  device, 256-byte aligned, >= aoh_head_classify_workspace_size
 * A key block without full row rank has no Cholesky factor: the ER of its
 * q heads is NaN and device check 5 is recorded.
 */
aoh_status aoh_head_classify(const void* w_q, const void* w_k, int32_t d_model, int32_t n_q_heads,
                             int32_t n_kv_heads, int32_t head_dim, int32_t n_retrieval,
                             double* er_heads, double* er_groups, uint8_t* roles, void* workspace,
                             size_t workspace_bytes, void* stream);

size_t aoh_head_classify_workspace_size(int32_t d_model, int32_t n_q_heads, int32_t n_kv_heads,
                                        int32_t head_dim);

/*
 * FASA-M, the memory-saving variant (FASA section 2.C): the value cache and
 * the non-dominant parts of the keys live in host memory; only the dominant
 * components of K stay on the GPU.  The importance scan and the top-N_fac
 * select run on the GPU part; only the selected tokens' rows cross the host
 * link.  Head-major layouts, token t of KV head g:
 *   k_dom   device bf16 [n_kv_heads][total_tokens][k_dom_cols]: the packed
 *           dominant columns of aoh_kv_cache (dims I_dom, then I_dom + d/2)
 *   k_rest  host bf16 [n_kv_heads][total_tokens][rest_cols]: the other
 *           d - 2 n_dom dims in ascending order, zero-padded to rest_cols
 *   v       host bf16 [n_kv_heads][total_tokens][head_dim]
 * Host buffers must be pinned (page-locked, e.g. cudaHostAlloc) so the GPU can
 * read them in place; pageable memory is refused (AOH_ERR_INVALID_ARG).
 * offsets / lengths: as in aoh_kv_cache.  Every KV head is SPARSE here.
 * I_dom sizes must be multiples of 4 (whole 16-byte dominant segments).
 */
typedef struct aoh_offload_cache {
  const int32_t* offsets;      /* device int32 [batch + 1]                             */
  const int32_t* lengths;      /* device int32 [batch] or NULL                         */
  int32_t batch;
  int32_t n_kv_heads;          /* 1..128                                               */
  int32_t head_dim;            /* 64 or 128                                            */
  int32_t max_len;             /* host upper bound of the lengths                      */
  int64_t total_tokens;        /* host copy of offsets[batch], < 2^31                  */
  const void* k_dom;           /* device, 16-byte aligned                              */
  int32_t k_dom_cols;          /* multiple of 8, >= 2 n_dom                            */
  int32_t rest_cols;           /* multiple of 8, >= head_dim - 2 n_dom, <= head_dim     */
  const void* k_rest;          /* pinned host, 16-byte aligned                         */
  const void* v;               /* pinned host, 16-byte aligned                         */
} aoh_offload_cache;

/*
 * aoh_offload_split -- write the host parts (k_rest, v) of every head from a
 * linear device cache `kv` (every head stored), with I_dom of n_dom chunks per
 * head; rows are written over the host link.  Cache maintenance, not a decode
 * step.  k_dom is written by aoh_pack_dominant.
 */
aoh_status aoh_offload_split(const aoh_kv_cache* kv, const int32_t* idom, int32_t n_dom,
                             void* k_rest, int32_t rest_cols, void* v, void* stream);

/*
 * aoh_offload_decode -- aoh_sparse_decode on a FASA-M cache: the scan of k_dom
 * and the select on the GPU, then the K rows (dominant part from k_dom, the
 * rest from the host) and V rows of the selected tokens are brought across
 * the link into the workspace, and focused attention runs on them.  The K rows
 * and q are taken in each head's dominant-first dim order, which leaves every
 * q.k unchanged.  Arguments as for aoh_sparse_decode (every head SPARSE);
 * workspace >= aoh_offload_decode_workspace_size, zero-filled before first use.
 */
aoh_status aoh_offload_decode(const void* q, int32_t n_q_heads, const aoh_offload_cache* oc,
                              const int32_t* idom, int32_t n_dom, int32_t n_fac,
                              const int32_t* n_fac_per_seq, int32_t n_fac_cap, float scale,
                              float* out, int32_t* idx_out, int32_t* count_out, void* workspace,
                              size_t workspace_bytes, void* stream);

size_t aoh_offload_decode_workspace_size(const aoh_offload_cache* oc, int32_t n_q_heads,
                                         int32_t n_fac_cap);

#ifdef __cplusplus
}
#endif

#endif /* AOH_H */
