// C ABI of the token-sparse decode step: argument checks on the host, then
// asynchronous launches on the caller's stream.  Declarations and the contract
// of every entry point are in include/aoh.h.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "aoh.h"
#include "device_common.cuh"
#include "flash_gather.cuh"
#include "head_classify.cuh"
#include "kv_append.cuh"
#include "offload.cuh"
#include "select_cluster.cuh"
#include "select_hist.cuh"
#include "sparse_row.cuh"
#include "tip_score.cuh"

using namespace aoh;

namespace {

constexpr int kMaxQRows = 32;        // query rows per KV head in one gather kernel (4 n-tiles)

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

aoh_status check_kv(const aoh_kv_cache* kv) {
  if (!kv) return AOH_ERR_INVALID_ARG;
  if (kv->batch < 0 || kv->n_kv_heads < 1 || kv->n_kv_heads > kMaxHeads) return AOH_ERR_INVALID_ARG;
  if (kv->head_dim != 64 && kv->head_dim != 128) return AOH_ERR_UNSUPPORTED;
  if (kv->max_len < 0 || kv->total_tokens < 0 || kv->total_tokens >= (int64_t(1) << 31))
    return AOH_ERR_INVALID_ARG;
  if (kv->batch == 0) return AOH_OK;
  if (!kv->k || !kv->v || !kv->offsets) return AOH_ERR_INVALID_ARG;
  if (kv->stride_tok < 1 || kv->stride_head < 1) return AOH_ERR_INVALID_ARG;
  if (!aligned16(kv->k) || !aligned16(kv->v) || (kv->stride_tok % 8) || (kv->stride_head % 8))
    return AOH_ERR_ALIGNMENT;
  if (kv->k_dom) {
    if (kv->k_dom_cols < 8 || kv->k_dom_cols > 128 || (kv->k_dom_cols % 8)) return AOH_ERR_INVALID_ARG;
    if (!aligned16(kv->k_dom)) return AOH_ERR_ALIGNMENT;
  }
  if (kv->ring_sink < 0 || kv->ring_window < 0) return AOH_ERR_INVALID_ARG;
  return AOH_OK;
}

bool is_ring(const aoh_kv_cache* kv) { return kv->ring_sink + kv->ring_window > 0; }

// KV head g's slot in this cache's K / V (and k_dom), or kNoSlot when the cache does not store it
uint8_t slot_of(const aoh_kv_cache* kv, int g) { return kv->head_slot ? kv->head_slot[g] : (uint8_t)g; }

// per-sequence lengths and head slots of the cache, into any kernel's parameters
template <typename P>
void bind_cache(P& prm, const aoh_kv_cache* kv) {
  prm.lengths = kv->lengths;
  for (int g = 0; g < kv->n_kv_heads; ++g) prm.slot[g] = slot_of(kv, g);
}

aoh_status check_heads(const aoh_kv_cache* kv, int32_t n_q_heads) {
  if (n_q_heads < 1 || n_q_heads % kv->n_kv_heads) return AOH_ERR_INVALID_ARG;
  return AOH_OK;
}

thread_local int t_last_cuda_error = 0;

// Streaming multiprocessors of the current device (148 on a B200), read once per device.
// Grids of the persistent and split-K kernels are sized from it.
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  std::atomic<int>& slot = cached[dev & 63];
  int n = slot.load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 148;
  }
  slot.store(n, std::memory_order_relaxed);
  return n;
}


aoh_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return AOH_OK;
  t_last_cuda_error = (int)e;
  return AOH_ERR_CUDA;
}

std::atomic<int64_t> g_launches[AOH_KERNEL_KINDS];

// aoh_record_launch_events state: events[0] before the first launch, events[i] after launch i
struct LaunchEvents {
  cudaEvent_t* ev = nullptr;
  int32_t* kinds = nullptr;
  int n = 0;
  int next = 0;
};
LaunchEvents g_ev;

void before_launch(cudaStream_t st) {
  if (g_ev.ev && g_ev.next == 0 && g_ev.n > 1) {
    cudaEventRecord(g_ev.ev[0], st);
    g_ev.next = 1;
  }
}

// status of the launch just made on `st`; counts it under `kind` when the runtime accepted it
aoh_status count_launch(aoh_kernel_kind kind, cudaStream_t st) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e);
  g_launches[kind].fetch_add(1, std::memory_order_relaxed);
  if (g_ev.ev && g_ev.next > 0 && g_ev.next < g_ev.n) {
    if (g_ev.kinds) g_ev.kinds[g_ev.next - 1] = kind;
    cudaEventRecord(g_ev.ev[g_ev.next++], st);
  }
  return AOH_OK;
}

// Opt in to `bytes` of dynamic shared memory.  Always set: static shared memory
// counts against the 48 KB default too.
template <typename F>
aoh_status set_smem(F* kernel, size_t bytes) {
  return cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
}

// One-time set-up per device: function attributes apply to the current device only, so a
// process that drives several GPUs sets them once on each.  `done` is a per-call-site mask
// of device ordinals (devices 0..63).
inline bool set_up_on_this_device(std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  return (done.load(std::memory_order_acquire) >> (dev & 63)) & 1ull;
}
inline void mark_set_up(std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  done.fetch_or(1ull << (dev & 63), std::memory_order_release);
}

// ------------------------------------------------------------------ gather-kernel geometry
struct FdGeom {
  int chunk;
  int max_splits;
  int nqp;
  int rows;     // partial-state rows: sequences x KV heads x q_split
  int q_split;  // CTAs sharing a row's positions, each with nqp of its query rows
  size_t ticket_bytes, ml_bytes, acc_bytes;
};

FdGeom fd_geom(int64_t work_tokens, int64_t n_max, int rows, int nq, int d) {
  FdGeom g{};
  // about two CTAs per SM; at least two pipeline stages per CTA; at most kFdMaxSplits splits a row
  const int64_t target = int64_t(sm_count()) * 2;
  int64_t chunk = ceil_div(std::max<int64_t>(work_tokens, 1), target);
  chunk = std::min<int64_t>(std::max<int64_t>(chunk, 2 * kFdTS), 1024);  // long CTAs are latency bound
  chunk = std::max<int64_t>(chunk, ceil_div(std::max<int64_t>(n_max, 1), kFdMaxSplits));
  chunk = ceil_div(chunk, kFdTS) * kFdTS;
  g.nqp = nq <= 8 ? 8 : (nq <= 16 ? 16 : 32);
  // partials grow with the query rows and the last CTA of a row reads them all: at most 16
  // splits for 16 query rows, 8 for 32 (measured: 16 splits of the 32-row shared-index gather,
  // merged in 16-CTA clusters, took 32.9 us against 24.9 us for 8)
  if (g.nqp > 8) {
    const int64_t max_sp = g.nqp == 16 ? 16 : 8;
    chunk = std::max<int64_t>(chunk, ceil_div(ceil_div(std::max<int64_t>(n_max, 1), max_sp), kFdTS) * kFdTS);
  }
  g.chunk = (int)chunk;
  g.max_splits = (int)std::max<int64_t>(1, ceil_div(std::max<int64_t>(n_max, 1), chunk));
  g.rows = rows;
  g.q_split = 1;
  g.ticket_bytes = align256(sizeof(int32_t) * (size_t)std::max(rows, 1));
  g.ml_bytes = align256(sizeof(float) * (size_t)rows * g.max_splits * g.nqp * 2);
  g.acc_bytes = align256(sizeof(float) * (size_t)rows * g.max_splits * g.nqp * d);
  return g;
}

size_t fd_bytes(const FdGeom& g) { return g.ticket_bytes + g.ml_bytes + g.acc_bytes; }

// Workspace layout: [tickets][part_ml][part_acc][extra...]; tickets first so that a
// zero-filled workspace starts with zero tickets.
void fd_bind(FdecParams& fp, const FdGeom& g, uint8_t* ws) {
  fp.tickets = reinterpret_cast<int32_t*>(ws);
  fp.part_ml = reinterpret_cast<float*>(ws + g.ticket_bytes);
  fp.part_acc = reinterpret_cast<float*>(ws + g.ticket_bytes + g.ml_bytes);
  fp.chunk = g.chunk;
  fp.max_splits = g.max_splits;
  fp.q_split = g.q_split;
}

// Launch of a kernel that follows another one of the same call on the stream: programmatic
// dependent launch lets it be scheduled while that kernel drains (the kernel itself waits for
// it with griddepcontrol.wait before touching memory); cl > 0 adds a cluster dimension.
constexpr int kDependentLaunch = 1;

template <typename K, typename P>
aoh_status launch_dependent(K kern, dim3 grid, int threads, size_t smem, int cl, cudaStream_t st, const P& params) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (cl > 0) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cl;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = kDependentLaunch;
  ++na;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  before_launch(st);
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, params));
}

template <typename K>
int max_active_clusters(K kern, int CL, size_t smem, int threads = kSrThreads) {
  // (cluster size, dynamic shared memory) -> cudaOccupancyMaxActiveClusters, cached per process
  static std::mutex mu;
  static int keys[64][3];  // kernel id, CL, smem / 256 << 8 | clusters (threads fixed per kernel)
  static int n_keys = 0;
  std::lock_guard<std::mutex> lock(mu);
  const int kid = (int)(reinterpret_cast<uintptr_t>(reinterpret_cast<const void*>(kern)) & 0x7fffffff);
  for (int i = 0; i < n_keys; ++i)
    if (keys[i][0] == kid && keys[i][1] == CL && keys[i][2] >> 8 == (int)(smem >> 8)) return keys[i][2] & 0xff;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, 1, 1);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  n = std::min(n, 255);
  if (n_keys < 64) {
    keys[n_keys][0] = kid;
    keys[n_keys][1] = CL;
    keys[n_keys][2] = (int)((smem >> 8) << 8) | n;
    ++n_keys;
  }
  return n;
}

template <int D, int NT>
aoh_status launch_fd_t(FdecParams fp, int n_listed, int B, bool uniform, cudaStream_t st) {
  const size_t smem = FdTile<D>::kSmem;
  auto kern = flash_gather_kernel<D, NT>;
  static std::atomic<uint64_t> configured{0};
  if (!set_up_on_this_device(configured)) {
    aoh_status s = set_smem(kern, smem);
    if (s != AOH_OK) return s;
    s = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    if (s != AOH_OK) return s;
    mark_set_up(configured);
  }
  const int QS = std::max(1, fp.q_split);
  dim3 grid(fp.max_splits, n_listed * QS, B);
  // rows of about equal length with 2..16 splits: one cluster per row, merged on chip
  const int CL = fp.max_splits;
  constexpr int threads = fd_threads(NT);
  const bool merge_on_chip =
      uniform && CL >= 2 && CL <= kFdMaxCluster && max_active_clusters(kern, CL, smem, threads) > 0;
  fp.cluster_combine = merge_on_chip ? 1 : 0;
  // rows with many splits and no cluster merge: the gather leaves partials and a second launch
  // combines them over many CTAs (one CTA merging up to 256 splits is latency-bound)
  fp.defer_merge = (!merge_on_chip && fp.max_splits > kFdMaxCluster) ? 1 : 0;
  aoh_status s = launch_dependent(kern, grid, threads, smem, merge_on_chip ? CL : 0, st, fp);
  if (s != AOH_OK) return s;
  if ((s = count_launch(AOH_KERNEL_FLASH_GATHER, st)) != AOH_OK || !fp.defer_merge) return s;
  constexpr int NQP = NT * 8;
  const dim3 mgrid((unsigned)ceil_div(int64_t(std::min(fp.NQ, NQP)) * (D / 4), kFmOut), n_listed * QS, B);
  const size_t msmem = sizeof(float) * 2 * (size_t)fp.max_splits * NQP;  // <= 2 x 256 x 32 floats
  static std::atomic<uint64_t> merge_configured{0};
  if (!set_up_on_this_device(merge_configured)) {
    if ((s = set_smem(flash_merge_kernel<D, NT>, sizeof(float) * 2 * kFdMaxSplits * NQP)) != AOH_OK) return s;
    mark_set_up(merge_configured);
  }
  if ((s = launch_dependent(flash_merge_kernel<D, NT>, mgrid, kFmThreads, msmem, 0, st, fp)) != AOH_OK) return s;
  return count_launch(AOH_KERNEL_FLASH_MERGE, st);
}

// `uniform`: every row attends to about the same number of positions (a fixed N_fac or k)
aoh_status launch_fd(const FdecParams& fp, int d, int nqp, int n_listed, int B, cudaStream_t st,
                     bool uniform = false) {
  if (d == 128) {
    if (nqp == 8) return launch_fd_t<128, 1>(fp, n_listed, B, uniform, st);
    if (nqp == 16) return launch_fd_t<128, 2>(fp, n_listed, B, uniform, st);
    return launch_fd_t<128, 4>(fp, n_listed, B, uniform, st);
  }
  if (nqp == 8) return launch_fd_t<64, 1>(fp, n_listed, B, uniform, st);
  if (nqp == 16) return launch_fd_t<64, 2>(fp, n_listed, B, uniform, st);
  return launch_fd_t<64, 4>(fp, n_listed, B, uniform, st);
}

// ------------------------------------------------------------------ TIP scan
template <int S>
aoh_status launch_tip_t(TipParams& tp, cudaStream_t st) {
  static int per_sm = 0;  // resident CTAs per SM (cached per process)
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tip_score_kernel<S>, kTipThreads, 0) != cudaSuccess ||
        per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
  }
  const int64_t resident = int64_t(sm_count()) * per_sm;
  tp.per_cta = std::max<int64_t>(256, ceil_div(tp.total, resident));
  const int64_t grid = ceil_div(tp.total, tp.per_cta);
  before_launch(st);
  tip_score_kernel<S><<<(unsigned)grid, kTipThreads, 0, st>>>(tp);
  return count_launch(AOH_KERNEL_TIP_SCORE, st);
}

aoh_status launch_tip(const void* q, int32_t Hq, const aoh_kv_cache* kv, const int32_t* idom, int32_t n_dom,
                      float* scores, const uint8_t* heads, int n_listed, cudaStream_t st) {
  TipParams tp{};
  tp.q = static_cast<const uint16_t*>(q);
  tp.idom = idom;
  tp.offsets = kv->offsets;
  bind_cache(tp, kv);
  tp.scores = scores;
  tp.T = (int32_t)kv->total_tokens;
  tp.Hq = Hq;
  tp.Hkv = kv->n_kv_heads;
  tp.d = kv->head_dim;
  tp.G = Hq / kv->n_kv_heads;
  tp.n_dom = n_dom;
  const bool packed = kv->k_dom && idom;
  if (packed && 2 * n_dom > kv->k_dom_cols) return AOH_ERR_INVALID_ARG;
  if (packed) {
    tp.src = static_cast<const uint16_t*>(kv->k_dom);
    tp.row_stride_tok = kv->k_dom_cols;
    tp.row_stride_head = kv->total_tokens * kv->k_dom_cols;
    tp.row_len = kv->k_dom_cols;
    tp.packed = 1;
  } else {
    tp.src = static_cast<const uint16_t*>(kv->k);
    tp.row_stride_tok = kv->stride_tok;
    tp.row_stride_head = kv->stride_head;
    tp.row_len = kv->head_dim;
    tp.packed = 0;
  }
  memcpy(tp.heads, heads, n_listed);
  tp.B = kv->batch;
  tp.total = int64_t(n_listed) * kv->total_tokens;
  if (tp.total == 0) return AOH_OK;
  int lanes = 1;
  while (lanes * 8 < tp.row_len) lanes <<= 1;
  switch (lanes) {
    case 1: return launch_tip_t<1>(tp, st);
    case 2: return launch_tip_t<2>(tp, st);
    case 4: return launch_tip_t<4>(tp, st);
    case 8: return launch_tip_t<8>(tp, st);
    default: return launch_tip_t<16>(tp, st);
  }
}

// Full-dimension scores (every chunk; the shared indexer's score), K read in place.
aoh_status launch_tip_full(const void* q, int32_t Hq, const aoh_kv_cache* kv, float* scores, const uint8_t* heads,
                           int n_listed, cudaStream_t st) {
  return launch_tip(q, Hq, kv, nullptr, kv->head_dim / 2, scores, heads, n_listed, st);
}

// ------------------------------------------------------------------ chunked select
// Workspace of the select (after the scores): the histograms first (they must start at zero
// and every select leaves them at zero), then the candidate counts and list, the chunk counts
// and the row results.
struct SelectWs {
  size_t hist, cand_count, cand, chunk_above, chunk_info, row_info, total;
  int max_chunks;
};

SelectWs select_ws(const aoh_kv_cache* kv) {
  SelectWs w{};
  const size_t rows = (size_t)kv->n_kv_heads * (size_t)std::max(kv->batch, 1);
  w.max_chunks = (int)std::max<int64_t>(1, ceil_div(std::max(kv->max_len, 1), kSelChunk));
  size_t o = 0;
  w.hist = o;
  o += align256(rows * kSelHistBins * sizeof(uint32_t));
  w.cand_count = o;
  o += align256(rows * sizeof(int32_t));
  w.cand = o;
  o += align256((size_t)kv->n_kv_heads * (size_t)std::max<int64_t>(kv->total_tokens, 1) * sizeof(unsigned long long));
  w.chunk_above = o;
  o += align256(rows * w.max_chunks * sizeof(int32_t));
  w.chunk_info = o;
  o += align256(rows * w.max_chunks * 2 * sizeof(int32_t));
  w.row_info = o;
  o += align256(rows * kRowInfo * sizeof(int32_t));
  w.total = o;
  return w;
}

bool select_fits(const aoh_kv_cache* kv) { return ceil_div(std::max(kv->max_len, 1), kSelChunk) <= kSelMaxChunks; }

// The chunked select on the scores: histograms, chunk pass, resolve, ordered write (one
// launch per phase).  `ws` is the select's region (layout of select_ws).
aoh_status launch_chunk_select(const float* scores, const aoh_kv_cache* kv, int32_t n_fac, const int32_t* nfps,
                               int32_t cap, int32_t* idx, int32_t* count, const uint8_t* heads, int n_listed,
                               uint8_t* ws, cudaStream_t st) {
  if (!select_fits(kv)) return AOH_ERR_UNSUPPORTED;
  const SelectWs w = select_ws(kv);
  HistSelectParams hp{};
  hp.scores = scores;
  hp.offsets = kv->offsets;
  hp.lengths = kv->lengths;
  hp.n_fac_per_seq = nfps;
  hp.hist = reinterpret_cast<uint32_t*>(ws + w.hist);
  hp.cand = reinterpret_cast<unsigned long long*>(ws + w.cand);
  hp.cand_count = reinterpret_cast<int32_t*>(ws + w.cand_count);
  hp.chunk_above = reinterpret_cast<int32_t*>(ws + w.chunk_above);
  hp.chunk_info = reinterpret_cast<int32_t*>(ws + w.chunk_info);
  hp.row_info = reinterpret_cast<int32_t*>(ws + w.row_info);
  hp.idx = idx;
  hp.count = count;
  hp.T = (int32_t)kv->total_tokens;
  hp.B = kv->batch;
  hp.Hkv = kv->n_kv_heads;
  hp.n_fac = n_fac;
  hp.cap = cap;
  hp.max_chunks = w.max_chunks;
  memcpy(hp.heads, heads, n_listed);
  const dim3 grid(w.max_chunks, n_listed, kv->batch);
  aoh_status s;
  if (kv->total_tokens > 0) {
    if ((s = launch_dependent(select_hist_kernel, grid, kSelCtaThreads, 0, 0, st, hp)) != AOH_OK) return s;
    if ((s = count_launch(AOH_KERNEL_SELECT_HIST, st)) != AOH_OK) return s;
  }
  if ((s = launch_dependent(select_chunk_kernel, grid, kSelCtaThreads, 0, 0, st, hp)) != AOH_OK) return s;
  if ((s = count_launch(AOH_KERNEL_SELECT_CHUNK, st)) != AOH_OK) return s;
  if ((s = launch_dependent(select_resolve_kernel, dim3(1, n_listed, kv->batch), kSelCtaThreads, 0, 0, st, hp)) !=
      AOH_OK)
    return s;
  if ((s = count_launch(AOH_KERNEL_SELECT_RESOLVE, st)) != AOH_OK) return s;
  if ((s = launch_dependent(select_write_kernel, grid, kSelCtaThreads, 0, 0, st, hp)) != AOH_OK) return s;
  return count_launch(AOH_KERNEL_SELECT_WRITE, st);
}

// Cluster size of the on-chip select: the smallest power of two whose slices of
// kScSlice positions hold the longest row; 0 when none does.
int select_cluster_size(const aoh_kv_cache* kv) {
  const int64_t L = std::max(kv->max_len, 1);
  for (int cl = 1; cl <= kScMaxCluster; cl *= 2)
    if (L <= int64_t(cl) * kScSlice) return cl;
  return 0;
}

// The select on the scores: one cluster per row, on chip, when every row's cluster runs in
// one wave; else the chunked select, which spreads every row over all SMs (measured: the
// 128K shared-index rows, whose 16 clusters of 16 CTAs need two waves, and the 256 serving
// rows select faster chunked; 32 rows of 32K faster in clusters).  Both take the same
// workspace region.
aoh_status launch_select_rows(const float* scores, const aoh_kv_cache* kv, int32_t n_fac, const int32_t* nfps,
                              int32_t cap, int32_t* idx, int32_t* count, const uint8_t* heads, int n_listed,
                              cudaStream_t st, bool* launched);

aoh_status launch_select(const float* scores, const aoh_kv_cache* kv, int32_t n_fac, const int32_t* nfps, int32_t cap,
                         int32_t* idx, int32_t* count, const uint8_t* heads, int n_listed, uint8_t* ws,
                         cudaStream_t st) {
  const int CL = select_cluster_size(kv);
  const int64_t n_rows = int64_t(n_listed) * kv->batch;
  bool one_wave = false;
  if (CL > 0) {
    auto kern = select_cluster_kernel;
    static std::atomic<uint64_t> configured{0};
    if (!set_up_on_this_device(configured)) {
      const aoh_status s = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
      if (s != AOH_OK) return s;
      mark_set_up(configured);
    }
    const int maxc = max_active_clusters(kern, CL, 0, kScThreads);
    one_wave = maxc > 0 && n_rows <= maxc;
    if (one_wave) {
      ClusterSelectParams cp{};
      cp.scores = scores;
      cp.offsets = kv->offsets;
      cp.lengths = kv->lengths;
      cp.n_fac_per_seq = nfps;
      cp.idx = idx;
      cp.count = count;
      cp.T = (int32_t)kv->total_tokens;
      cp.Hkv = kv->n_kv_heads;
      cp.n_fac = n_fac;
      cp.cap = cap;
      memcpy(cp.heads, heads, n_listed);
      const aoh_status s = launch_dependent(kern, dim3(CL, n_listed, kv->batch), kScThreads, 0, CL, st, cp);
      if (s != AOH_OK) return s;
      return count_launch(AOH_KERNEL_SELECT_CLUSTER, st);
    }
  }
  // Fewer rows than SMs that the cluster select cannot take in one wave: the row kernel's
  // select over a cluster's shared memory (one launch, 8-bit digits), when its clusters fit.
  if (n_rows < sm_count()) {
    bool launched = false;
    const aoh_status s = launch_select_rows(scores, kv, n_fac, nfps, cap, idx, count, heads, n_listed, st, &launched);
    if (s != AOH_OK || launched) return s;
  }
  return launch_chunk_select(scores, kv, n_fac, nfps, cap, idx, count, heads, n_listed, ws, st);
}

// ------------------------------------------------------------------ fused row kernel
// Shared memory per CTA: keys of the slice, then a ring region used by the scan's
// per-warp cp.async rings (64 KB) and then by the attention stages.  Two CTAs per SM
// when the keys leave room for a ring of >= 64 KB in 108 KB, else one CTA per SM with
// up to 128 KB of ring (sized in 16 KB steps).
constexpr size_t kTwoPerSm = 108 * 1024;
constexpr size_t kOnePerSm = 220 * 1024;
constexpr size_t kRingStep = 16 * 1024;
constexpr size_t kRingMin = kSrRingMin;
constexpr size_t kRingMax = 8 * kRingStep;
constexpr int kShortRow = 2048;  // rows this short run as one CTA each (no cluster exchange)

struct FusedPlan {
  bool ok;
  int CL;
  int slice;
  size_t keys_bytes, ring_bytes, smem;
};

FusedPlan fused_candidate(const aoh_kv_cache* kv, int CL, bool select_only = false) {
  FusedPlan f{};
  const int64_t L = std::max(kv->max_len, 1);
  const int64_t slice = (ceil_div(L, CL) + 3) & ~int64_t(3);
  if (slice > int64_t(kSrThreads) * kSrMaxRun) return f;  // row too long for CL CTAs
  f.CL = CL;
  f.slice = (int)slice;
  f.keys_bytes = (size_t)ceil_div(slice * 4, 1024) * 1024;
  if (select_only) {
    // no scan ring and no attention stages: the ring region only holds the candidates of the
    // first digit (more than fit are re-read from the keys), so CTAs stay small and many fit an SM
    f.ring_bytes = kRingStep;
    f.smem = f.keys_bytes + f.ring_bytes + 1024;
    f.ok = true;
    return f;
  }
  // 1 KB of slack: the kernel aligns its dynamic shared memory to 1024 bytes
  size_t budget = kTwoPerSm - 1024;
  const size_t ring_min = kRingMin;
  if (f.keys_bytes + ring_min > budget) budget = kOnePerSm - 1024;
  if (f.keys_bytes + ring_min > budget) return f;
  f.ring_bytes = std::min(kRingMax, (budget - f.keys_bytes) / kRingStep * kRingStep);
  f.smem = f.keys_bytes + f.ring_bytes + 1024;
  f.ok = true;
  return f;
}

// The fused scan shares a row among cols / 8 lanes: a power of two from 16 columns.
bool packed_scan(const aoh_kv_cache* kv, const int32_t* idom) {
  const int c = kv->k_dom_cols;
  return kv->k_dom && idom && c >= 16 && (c & (c - 1)) == 0;
}

// Whether some cluster size handles these rows in one fused launch.
bool fused_feasible(const aoh_kv_cache* kv, int nq) {
  return nq <= kMaxQRows && fused_candidate(kv, kSrMaxCluster).ok;
}



// Launch the cluster row kernel with the cluster size that needs the fewest waves x slice
// length (ties to the smaller cluster).  With max_waves > 0 nothing is launched when every
// choice needs more waves; *launched says which happened.
template <int D, int NT, bool SO = false>
aoh_status launch_rows_t(RowParams rp, const aoh_kv_cache* kv, int n_listed, int B, cudaStream_t st, int max_waves,
                         bool* launched) {
  *launched = false;
  auto kern = sparse_row_kernel<D, NT, SO>;
  static std::atomic<uint64_t> configured{0};
  if (!set_up_on_this_device(configured)) {
    aoh_status s = set_smem(kern, kOnePerSm);
    if (s != AOH_OK) return s;
    s = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    if (s != AOH_OK) return s;
    mark_set_up(configured);
  }
  const int n_rows = n_listed * B;
  FusedPlan best{};
  int64_t best_cost = INT64_MAX, best_waves = 0;
  // Short rows (<= kShortRow positions) take one CTA per row when that fits one wave: their
  // time is the fixed cost of the phases, and a one-CTA cluster's barriers are block barriers.
  if (kv->max_len <= kShortRow) {
    const FusedPlan f = fused_candidate(kv, 1, SO);
    if (f.ok) {
      const int maxc = max_active_clusters(kern, 1, f.smem);
      if (maxc > 0 && n_rows <= maxc) {
        best = f;
        best_waves = 1;
        best_cost = 0;
      }
    }
  }
  const int cls[3] = {4, 8, 16};
  for (int i = 0; i < 3 && best_cost > 0; ++i) {
    const FusedPlan f = fused_candidate(kv, cls[i], SO);
    if (!f.ok) continue;
    const int maxc = max_active_clusters(kern, f.CL, f.smem);
    if (maxc <= 0) continue;
    const int64_t waves = ceil_div(n_rows, maxc);
    const int64_t cost = waves * f.slice;
    if (cost < best_cost) {
      best_cost = cost;
      best_waves = waves;
      best = f;
    }
  }
  if (!best.ok) return AOH_ERR_UNSUPPORTED;
  if (max_waves > 0 && best_waves > max_waves) return AOH_OK;
  rp.keys_bytes = (int32_t)best.keys_bytes;
  rp.ring_bytes = (int32_t)best.ring_bytes;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(best.CL, n_listed, B);
  cfg.blockDim = dim3(kSrThreads);
  cfg.dynamicSmemBytes = best.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = best.CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  before_launch(st);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, rp);
  const aoh_status s = e != cudaSuccess ? cuda_status(e) : count_launch(AOH_KERNEL_SPARSE_ROW, st);
  *launched = (s == AOH_OK);
  return s;
}

aoh_status launch_rows(const RowParams& rp, const aoh_kv_cache* kv, int nq, int n_listed, int B, cudaStream_t st,
                       int max_waves, bool* launched) {
  const int nqp = nq <= 8 ? 8 : (nq <= 16 ? 16 : 32);
  if (kv->head_dim == 128) {
    if (nqp == 8) return launch_rows_t<128, 1>(rp, kv, n_listed, B, st, max_waves, launched);
    if (nqp == 16) return launch_rows_t<128, 2>(rp, kv, n_listed, B, st, max_waves, launched);
    return launch_rows_t<128, 4>(rp, kv, n_listed, B, st, max_waves, launched);
  }
  if (nqp == 8) return launch_rows_t<64, 1>(rp, kv, n_listed, B, st, max_waves, launched);
  if (nqp == 16) return launch_rows_t<64, 2>(rp, kv, n_listed, B, st, max_waves, launched);
  return launch_rows_t<64, 4>(rp, kv, n_listed, B, st, max_waves, launched);
}

// Select-only launch of the row kernel on the stand-alone scan's scores: writes idx / count.
// Nothing is launched (*launched false) when no cluster size takes the rows in one wave.
aoh_status launch_select_rows(const float* scores, const aoh_kv_cache* kv, int32_t n_fac, const int32_t* nfps,
                              int32_t cap, int32_t* idx, int32_t* count, const uint8_t* heads, int n_listed,
                              cudaStream_t st, bool* launched) {
  *launched = false;
  if (!fused_candidate(kv, kSrMaxCluster, true).ok) return AOH_OK;
  RowParams rp{};
  rp.offsets = kv->offsets;
  rp.lengths = kv->lengths;
  rp.scores_in = scores;
  rp.n_fac_per_seq = nfps;
  rp.n_fac = n_fac;
  rp.cap = cap;
  rp.idx_out = idx;
  rp.count_out = count;
  rp.T = (int32_t)kv->total_tokens;
  rp.B = kv->batch;
  rp.Hkv = kv->n_kv_heads;
  rp.G = 1;
  rp.NQ = 1;
  memcpy(rp.heads, heads, n_listed);
  return launch_rows_t<128, 1, true>(rp, kv, n_listed, kv->batch, st, 1, launched);
}

// Score source of the fused kernel: packed dominant columns, K in place masked to I_dom,
// or (idom == nullptr) K in place with every chunk.
void rows_score_source(RowParams& rp, const aoh_kv_cache* kv, const int32_t* idom, int32_t n_dom) {
  rp.idom = idom;
  rp.n_dom = n_dom;
  if (packed_scan(kv, idom)) {
    rp.score_src = static_cast<const uint16_t*>(kv->k_dom);
    rp.srow_stride_tok = kv->k_dom_cols;
    rp.srow_stride_head = kv->total_tokens * kv->k_dom_cols;
    rp.srow_len = kv->k_dom_cols;
    rp.packed = 1;
  } else {
    rp.score_src = static_cast<const uint16_t*>(kv->k);
    rp.srow_stride_tok = kv->stride_tok;
    rp.srow_stride_head = kv->stride_head;
    rp.srow_len = kv->head_dim;
    rp.packed = 0;
  }
}

// The KV heads a call computes: those of its roles that this cache stores.
int list_heads(const aoh_kv_cache* kv, const uint8_t* roles, bool want_sparse, uint8_t* out) {
  int n = 0;
  for (int g = 0; g < kv->n_kv_heads; ++g) {
    const uint8_t r = roles ? roles[g] : (uint8_t)AOH_ROLE_SPARSE;
    const bool sparse = (r == AOH_ROLE_SPARSE);
    if (sparse == want_sparse && slot_of(kv, g) != kNoSlot) out[n++] = (uint8_t)g;
  }
  return n;
}

aoh_status check_roles(const aoh_kv_cache* kv, const uint8_t* roles) {
  if (!roles) return AOH_OK;
  for (int g = 0; g < kv->n_kv_heads; ++g)
    if (roles[g] > AOH_ROLE_STREAM) return AOH_ERR_INVALID_ARG;
  return AOH_OK;
}

// Geometry of the sparse step (depends only on what the size query also sees).
FdGeom sparse_geom(const aoh_kv_cache* kv, int32_t Hq, int32_t cap) {
  const int G = Hq / kv->n_kv_heads;
  const int rows = kv->batch * kv->n_kv_heads;
  return fd_geom(int64_t(rows) * cap, cap, rows, G, kv->head_dim);
}

size_t sparse_ws_bytes(const aoh_kv_cache* kv, int32_t Hq, int32_t cap, size_t* off_scores, size_t* off_idx,
                       size_t* off_count) {
  const FdGeom g = sparse_geom(kv, Hq, cap);
  size_t o = fd_bytes(g);
  *off_scores = o;
  o += align256(sizeof(float) * (size_t)kv->n_kv_heads * (size_t)kv->total_tokens);
  *off_idx = o;
  o += align256(sizeof(int32_t) * (size_t)kv->batch * kv->n_kv_heads * (size_t)cap);
  *off_count = o;
  o += align256(sizeof(int32_t) * (size_t)kv->batch * kv->n_kv_heads);
  return o + select_ws(kv).total;  // the select's region last
}

FdGeom stream_geom(const aoh_kv_cache* kv, int32_t Hq, const uint8_t* roles, int32_t sink, int32_t window) {
  int64_t n_max = 0, work = 0;
  for (int g = 0; g < kv->n_kv_heads; ++g) {
    const uint8_t r = roles[g];
    if (r == AOH_ROLE_SPARSE || slot_of(kv, g) == kNoSlot) continue;
    const int64_t L = kv->max_len;
    const int64_t n = (r == AOH_ROLE_DENSE) ? L : std::min<int64_t>(L, int64_t(sink) + window);
    n_max = std::max(n_max, n);
    work += n * kv->batch;
  }
  const int G = Hq / kv->n_kv_heads;
  return fd_geom(work, n_max, kv->batch * kv->n_kv_heads, G, kv->head_dim);
}

// More than 16 query rows (the layers x group of a shared index) are split over two CTAs that
// read the same positions: twice the CTAs, each with half the contraction and half the partials
// (measured on the 128K shared-index step's 32 rows: see the gather's notes).
FdGeom shared_geom(const aoh_kv_cache* kv, int32_t n_layers, int32_t Hq, int32_t cap) {
  const int G = Hq / kv->n_kv_heads;
  const int nq = n_layers * G;
  const int qs = nq > 16 ? 2 : 1;
  const int rows = kv->batch * kv->n_kv_heads * qs;
  FdGeom g = fd_geom(int64_t(rows) * cap, cap, rows, (nq + qs - 1) / qs, kv->head_dim);
  g.q_split = qs;
  return g;
}

// A ring keeps only streaming heads' sink and window: it serves STREAM heads whose sink and
// window lie within its own, and stores no DENSE head.
aoh_status check_ring_roles(const aoh_kv_cache* kv, const uint8_t* roles, int32_t sink, int32_t window) {
  if (!is_ring(kv)) return AOH_OK;
  if (sink > kv->ring_sink || window > kv->ring_window) return AOH_ERR_INVALID_ARG;
  for (int g = 0; g < kv->n_kv_heads; ++g)
    if (roles[g] == AOH_ROLE_DENSE && slot_of(kv, g) != kNoSlot) return AOH_ERR_INVALID_ARG;
  return AOH_OK;
}

bool ws_ok(const void* ws, size_t have, size_t need) {
  if (need == 0) return true;
  return ws && have >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0;
}

}  // namespace

// ===================================================================== exported
extern "C" {

const char* aoh_status_string(aoh_status s) {
  switch (s) {
    case AOH_OK: return "ok";
    case AOH_ERR_INVALID_ARG: return "invalid argument";
    case AOH_ERR_UNSUPPORTED: return "unsupported shape";
    case AOH_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case AOH_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case AOH_ERR_CUDA: return "CUDA error";
    case AOH_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

int32_t aoh_version(void) { return 2; }

int32_t aoh_last_cuda_error(void) { return t_last_cuda_error; }

void aoh_record_launch_events(void** events, int32_t* kinds, int32_t n) {
  g_ev.ev = reinterpret_cast<cudaEvent_t*>(events);
  g_ev.kinds = kinds;
  g_ev.n = events ? n : 0;
  g_ev.next = 0;
}

int32_t aoh_launch_counts(int64_t* counts, int32_t n) {
  for (int i = 0; i < n && i < AOH_KERNEL_KINDS && counts; ++i) counts[i] = g_launches[i].load(std::memory_order_relaxed);
  return AOH_KERNEL_KINDS;
}

aoh_status aoh_device_check(void* stream, int32_t* detail) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return AOH_ERR_CUDA;
  int h[4] = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(h, g_device_error, sizeof(h)) != cudaSuccess) return AOH_ERR_CUDA;
  if (detail) memcpy(detail, h, sizeof(h));
  if (h[0] == 0) return AOH_OK;
  const int z[4] = {0, 0, 0, 0};
  if (cudaMemcpyToSymbol(g_device_error, z, sizeof(z)) != cudaSuccess) return AOH_ERR_CUDA;
  return AOH_ERR_DEVICE_CHECK;
}

aoh_status aoh_pack_dominant(const aoh_kv_cache* kv, const int32_t* idom, int32_t n_dom, void* k_dom,
                             int32_t k_dom_cols, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if (n_dom < 1 || n_dom > kv->head_dim / 2) return AOH_ERR_INVALID_ARG;
  if (k_dom_cols < 2 * n_dom || k_dom_cols > 128 || (k_dom_cols % 8)) return AOH_ERR_INVALID_ARG;
  if (kv->batch == 0 || kv->total_tokens == 0) return AOH_OK;
  if (!idom || !k_dom) return AOH_ERR_INVALID_ARG;
  if (!aligned16(k_dom)) return AOH_ERR_ALIGNMENT;
  if (is_ring(kv)) return AOH_ERR_INVALID_ARG;
  PackParams pp{};
  pp.k = static_cast<const uint16_t*>(kv->k);
  pp.idom = idom;
  pp.k_dom = static_cast<uint16_t*>(k_dom);
  pp.stride_tok = kv->stride_tok;
  pp.stride_head = kv->stride_head;
  pp.T = (int32_t)kv->total_tokens;
  pp.d = kv->head_dim;
  pp.n_dom = n_dom;
  pp.cols = k_dom_cols;
  pp.n_listed = list_heads(kv, nullptr, true, pp.heads);  // every stored head (roles NULL: all SPARSE)
  for (int g = 0; g < kv->n_kv_heads; ++g) pp.slot[g] = slot_of(kv, g);
  if (pp.n_listed == 0) return AOH_OK;
  const int64_t total = int64_t(pp.n_listed) * pp.T * pp.cols;
  const int blocks = (int)std::min<int64_t>(ceil_div(total, 256), int64_t(sm_count()) * 16);
  before_launch(as_stream(stream));
  pack_dominant_kernel<<<blocks, 256, 0, as_stream(stream)>>>(pp);
  return count_launch(AOH_KERNEL_PACK_DOMINANT, as_stream(stream));
}

aoh_status aoh_tip_score(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv, const int32_t* idom,
                         int32_t n_dom, float* scores, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if (is_ring(kv)) return AOH_ERR_INVALID_ARG;  // a ring holds streaming heads only
  if ((s = check_heads(kv, n_q_heads)) != AOH_OK) return s;
  if (n_dom < 1 || n_dom > kv->head_dim / 2) return AOH_ERR_INVALID_ARG;
  if (kv->batch == 0 || kv->total_tokens == 0) return AOH_OK;
  if (!q || !idom || !scores) return AOH_ERR_INVALID_ARG;
  uint8_t heads[kMaxHeads];
  const int n = list_heads(kv, nullptr, true, heads);
  return launch_tip(q, n_q_heads, kv, idom, n_dom, scores, heads, n, as_stream(stream));
}

size_t aoh_topk_select_workspace_size(const aoh_kv_cache* kv) {
  if (check_kv(kv) != AOH_OK || is_ring(kv)) return 0;
  return select_ws(kv).total;
}

aoh_status aoh_topk_select(const float* scores, const aoh_kv_cache* kv, int32_t n_fac,
                           const int32_t* n_fac_per_seq, int32_t n_fac_cap, int32_t* idx, int32_t* count,
                           void* workspace, size_t workspace_bytes, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if (is_ring(kv)) return AOH_ERR_INVALID_ARG;  // a ring holds streaming heads only
  if (n_fac_cap < 1) return AOH_ERR_INVALID_ARG;
  if (!n_fac_per_seq && (n_fac < 0 || n_fac > n_fac_cap)) return AOH_ERR_INVALID_ARG;
  if (kv->batch == 0) return AOH_OK;
  if (!idx || !count || (!scores && kv->total_tokens > 0)) return AOH_ERR_INVALID_ARG;
  if (!select_fits(kv)) return AOH_ERR_UNSUPPORTED;
  if (!ws_ok(workspace, workspace_bytes, select_ws(kv).total)) return AOH_ERR_WORKSPACE;
  uint8_t heads[kMaxHeads];
  const int n = list_heads(kv, nullptr, true, heads);
  return launch_select(scores, kv, n_fac, n_fac_per_seq, n_fac_cap, idx, count, heads, n,
                       static_cast<uint8_t*>(workspace), as_stream(stream));
}

size_t aoh_sparse_decode_workspace_size(const aoh_kv_cache* kv, int32_t n_q_heads, int32_t n_fac_cap) {
  if (check_kv(kv) != AOH_OK || check_heads(kv, n_q_heads) != AOH_OK || n_fac_cap < 1) return 0;
  if (n_q_heads / kv->n_kv_heads > kMaxQRows) return 0;
  size_t a, b, c;
  return sparse_ws_bytes(kv, n_q_heads, n_fac_cap, &a, &b, &c);
}

aoh_status aoh_sparse_decode(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv, const int32_t* idom,
                             int32_t n_dom, int32_t n_fac, const int32_t* n_fac_per_seq, int32_t n_fac_cap,
                             const uint8_t* roles, float scale, float* out, int32_t* idx_out,
                             int32_t* count_out, void* workspace, size_t workspace_bytes, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if (is_ring(kv)) return AOH_ERR_INVALID_ARG;  // a ring holds streaming heads only
  if ((s = check_heads(kv, n_q_heads)) != AOH_OK) return s;
  if ((s = check_roles(kv, roles)) != AOH_OK) return s;
  const int G = n_q_heads / kv->n_kv_heads;
  if (G > kMaxQRows) return AOH_ERR_UNSUPPORTED;
  if (n_dom < 1 || n_dom > kv->head_dim / 2) return AOH_ERR_INVALID_ARG;
  if (n_fac_cap < 1) return AOH_ERR_INVALID_ARG;
  if (!n_fac_per_seq && (n_fac < 0 || n_fac > n_fac_cap)) return AOH_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return AOH_ERR_INVALID_ARG;
  if ((idx_out == nullptr) != (count_out == nullptr)) return AOH_ERR_INVALID_ARG;
  if (kv->k_dom && 2 * n_dom > kv->k_dom_cols) return AOH_ERR_INVALID_ARG;
  if (kv->batch == 0) return AOH_OK;
  if (!q || !idom || !out) return AOH_ERR_INVALID_ARG;
  if (!aligned16(q)) return AOH_ERR_ALIGNMENT;
  size_t off_scores, off_idx, off_count;
  const size_t need = sparse_ws_bytes(kv, n_q_heads, n_fac_cap, &off_scores, &off_idx, &off_count);
  if (!ws_ok(workspace, workspace_bytes, need)) return AOH_ERR_WORKSPACE;
  uint8_t heads[kMaxHeads];
  const int n_listed = list_heads(kv, roles, true, heads);
  if (n_listed == 0) return AOH_OK;
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* scores = reinterpret_cast<float*>(ws + off_scores);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + off_idx);
  int32_t* cnt = count_out ? count_out : reinterpret_cast<int32_t*>(ws + off_count);

  if (fused_feasible(kv, G)) {
    RowParams rp{};
    rp.q_score = static_cast<const uint16_t*>(q);
    rp.q_attn = static_cast<const uint16_t*>(q);
    rp.k = static_cast<const uint16_t*>(kv->k);
    rp.v = static_cast<const uint16_t*>(kv->v);
    rp.offsets = kv->offsets;
    bind_cache(rp, kv);
    rows_score_source(rp, kv, idom, n_dom);
    rp.n_fac_per_seq = n_fac_per_seq;
    rp.n_fac = n_fac;
    rp.cap = n_fac_cap;
    rp.idx_out = idx;
    rp.count_out = cnt;
    rp.out = out;
    rp.stride_tok = kv->stride_tok;
    rp.stride_head = kv->stride_head;
    rp.T = (int32_t)kv->total_tokens;
    rp.B = kv->batch;
    rp.Hq = n_q_heads;
    rp.Hkv = kv->n_kv_heads;
    rp.G = G;
    rp.NQ = G;
    rp.scale_log2 = scale * 1.4426950408889634f;
    memcpy(rp.heads, heads, n_listed);
    // one launch when every row's cluster runs in a single wave
    bool launched = false;
    if ((s = launch_rows(rp, kv, G, n_listed, kv->batch, st, 1, &launched)) != AOH_OK) return s;
    if (launched) return AOH_OK;
  }

  // otherwise: the scan over all SMs, the select on the (L2-resident) scores, and the
  // split-K gather
  if (!select_fits(kv)) return AOH_ERR_UNSUPPORTED;
  uint8_t* sel_ws = ws + off_count + align256(sizeof(int32_t) * (size_t)kv->batch * kv->n_kv_heads);
  if (kv->total_tokens > 0) {
    if ((s = launch_tip(q, n_q_heads, kv, idom, n_dom, scores, heads, n_listed, st)) != AOH_OK) return s;
  }
  s = launch_select(scores, kv, n_fac, n_fac_per_seq, n_fac_cap, idx, cnt, heads, n_listed, sel_ws, st);
  if (s != AOH_OK) return s;

  const FdGeom geo = sparse_geom(kv, n_q_heads, n_fac_cap);
  FdecParams fp{};
  fp.q = static_cast<const uint16_t*>(q);
  fp.k = static_cast<const uint16_t*>(kv->k);
  fp.v = static_cast<const uint16_t*>(kv->v);
  fp.offsets = kv->offsets;
  bind_cache(fp, kv);
  fp.idx = idx;
  fp.count = cnt;
  fp.out = out;
  fp.stride_tok = kv->stride_tok;
  fp.stride_head = kv->stride_head;
  fp.B = kv->batch;
  fp.Hq = n_q_heads;
  fp.Hkv = kv->n_kv_heads;
  fp.G = G;
  fp.NQ = G;
  fp.cap = n_fac_cap;
  fp.list_mode = 1;
  fp.scale_log2 = scale * 1.4426950408889634f;
  memcpy(fp.heads, heads, n_listed);
  fd_bind(fp, geo, ws);
  return launch_fd(fp, kv->head_dim, geo.nqp, n_listed, kv->batch, st, n_fac_per_seq == nullptr);
}

size_t aoh_stream_decode_workspace_size(const aoh_kv_cache* kv, int32_t n_q_heads, const uint8_t* roles,
                                        int32_t sink, int32_t window) {
  if (check_kv(kv) != AOH_OK || check_heads(kv, n_q_heads) != AOH_OK || !roles) return 0;
  if (check_roles(kv, roles) != AOH_OK || sink < 0 || window < 0) return 0;
  if (n_q_heads / kv->n_kv_heads > kMaxQRows) return 0;
  return fd_bytes(stream_geom(kv, n_q_heads, roles, sink, window));
}

aoh_status aoh_stream_decode(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv, const uint8_t* roles,
                             int32_t sink, int32_t window, float scale, float* out, void* workspace,
                             size_t workspace_bytes, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if ((s = check_heads(kv, n_q_heads)) != AOH_OK) return s;
  if (!roles) return AOH_ERR_INVALID_ARG;
  if ((s = check_roles(kv, roles)) != AOH_OK) return s;
  const int G = n_q_heads / kv->n_kv_heads;
  if (G > kMaxQRows) return AOH_ERR_UNSUPPORTED;
  if (sink < 0 || window < 0 || !std::isfinite(scale)) return AOH_ERR_INVALID_ARG;
  if ((s = check_ring_roles(kv, roles, sink, window)) != AOH_OK) return s;
  if (kv->batch == 0) return AOH_OK;
  if (!q || !out) return AOH_ERR_INVALID_ARG;
  if (!aligned16(q)) return AOH_ERR_ALIGNMENT;
  const FdGeom geo = stream_geom(kv, n_q_heads, roles, sink, window);
  if (!ws_ok(workspace, workspace_bytes, fd_bytes(geo))) return AOH_ERR_WORKSPACE;
  uint8_t heads[kMaxHeads];
  const int n_listed = list_heads(kv, roles, false, heads);
  if (n_listed == 0) return AOH_OK;
  FdecParams fp{};
  fp.q = static_cast<const uint16_t*>(q);
  fp.k = static_cast<const uint16_t*>(kv->k);
  fp.v = static_cast<const uint16_t*>(kv->v);
  fp.offsets = kv->offsets;
  bind_cache(fp, kv);
  fp.out = out;
  fp.stride_tok = kv->stride_tok;
  fp.stride_head = kv->stride_head;
  fp.B = kv->batch;
  fp.Hq = n_q_heads;
  fp.Hkv = kv->n_kv_heads;
  fp.G = G;
  fp.NQ = G;
  fp.cap = 0;
  fp.list_mode = 0;
  fp.sink = sink;
  fp.window = window;
  fp.ring_sink = kv->ring_sink;
  fp.ring_window = kv->ring_window;
  fp.scale_log2 = scale * 1.4426950408889634f;
  memcpy(fp.heads, heads, n_listed);
  memcpy(fp.roles, roles, kv->n_kv_heads);
  fd_bind(fp, geo, static_cast<uint8_t*>(workspace));
  return launch_fd(fp, kv->head_dim, geo.nqp, n_listed, kv->batch, as_stream(stream));
}

size_t aoh_decode_step_workspace_size(const aoh_kv_cache* kv, int32_t n_q_heads, int32_t n_fac_cap,
                                      const uint8_t* roles, int32_t sink, int32_t window) {
  if (check_kv(kv) != AOH_OK || check_heads(kv, n_q_heads) != AOH_OK || n_fac_cap < 1 || sink < 0 || window < 0)
    return 0;
  if (check_roles(kv, roles) != AOH_OK || n_q_heads / kv->n_kv_heads > kMaxQRows) return 0;
  size_t a, b, c;
  const size_t sparse = is_ring(kv) ? 0 : sparse_ws_bytes(kv, n_q_heads, n_fac_cap, &a, &b, &c);
  return sparse + (roles ? fd_bytes(stream_geom(kv, n_q_heads, roles, sink, window)) : 0);
}

aoh_status aoh_decode_step(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv, const int32_t* idom,
                           int32_t n_dom, int32_t n_fac, const int32_t* n_fac_per_seq, int32_t n_fac_cap,
                           const uint8_t* roles, int32_t sink, int32_t window, float scale, float* out,
                           int32_t* idx_out, int32_t* count_out, void* workspace, size_t workspace_bytes,
                           void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if ((s = check_heads(kv, n_q_heads)) != AOH_OK) return s;
  if ((s = check_roles(kv, roles)) != AOH_OK) return s;
  const int G = n_q_heads / kv->n_kv_heads;
  if (G > kMaxQRows) return AOH_ERR_UNSUPPORTED;
  if (sink < 0 || window < 0 || !std::isfinite(scale) || n_fac_cap < 1) return AOH_ERR_INVALID_ARG;
  uint8_t sparse_heads[kMaxHeads], win_heads[kMaxHeads];
  const int n_sparse = list_heads(kv, roles, true, sparse_heads);
  const int n_win = roles ? list_heads(kv, roles, false, win_heads) : 0;
  if (is_ring(kv) && n_sparse) return AOH_ERR_INVALID_ARG;
  size_t a, b, c;
  const size_t sparse_need = is_ring(kv) ? 0 : sparse_ws_bytes(kv, n_q_heads, n_fac_cap, &a, &b, &c);
  const size_t win_need = roles ? fd_bytes(stream_geom(kv, n_q_heads, roles, sink, window)) : 0;
  if (kv->batch == 0) return AOH_OK;
  if (!ws_ok(workspace, workspace_bytes, sparse_need + win_need)) return AOH_ERR_WORKSPACE;
  // one launch for every head when the fused row kernel holds all rows in one wave and the
  // window heads' lists are about as long as a selection (long dense rows keep the split-K gather)
  int64_t win_max = 0;
  for (int i = 0; i < n_win; ++i)
    win_max = std::max<int64_t>(win_max, roles[win_heads[i]] == AOH_ROLE_DENSE
                                             ? kv->max_len : std::min<int64_t>(kv->max_len, int64_t(sink) + window));
  if (n_sparse > 0 && n_win > 0 && !is_ring(kv) && win_max <= 4 * int64_t(n_fac_cap) && fused_feasible(kv, G) && q &&
      idom && out && aligned16(q) && n_dom >= 1 && n_dom <= kv->head_dim / 2 &&
      (n_fac_per_seq || (n_fac >= 0 && n_fac <= n_fac_cap)) && (idx_out == nullptr) == (count_out == nullptr) &&
      !(kv->k_dom && 2 * n_dom > kv->k_dom_cols)) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    RowParams rp{};
    rp.q_score = static_cast<const uint16_t*>(q);
    rp.q_attn = static_cast<const uint16_t*>(q);
    rp.k = static_cast<const uint16_t*>(kv->k);
    rp.v = static_cast<const uint16_t*>(kv->v);
    rp.offsets = kv->offsets;
    bind_cache(rp, kv);
    rows_score_source(rp, kv, idom, n_dom);
    rp.n_fac_per_seq = n_fac_per_seq;
    rp.n_fac = n_fac;
    rp.cap = n_fac_cap;
    rp.idx_out = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + b);
    rp.count_out = count_out ? count_out : reinterpret_cast<int32_t*>(ws + c);
    rp.out = out;
    rp.stride_tok = kv->stride_tok;
    rp.stride_head = kv->stride_head;
    rp.T = (int32_t)kv->total_tokens;
    rp.B = kv->batch;
    rp.Hq = n_q_heads;
    rp.Hkv = kv->n_kv_heads;
    rp.G = G;
    rp.NQ = G;
    rp.scale_log2 = scale * 1.4426950408889634f;
    rp.sink = sink;
    rp.window = window;
    memcpy(rp.roles, roles, kv->n_kv_heads);
    uint8_t heads[kMaxHeads];
    memcpy(heads, sparse_heads, n_sparse);
    memcpy(heads + n_sparse, win_heads, n_win);
    memcpy(rp.heads, heads, n_sparse + n_win);
    bool launched = false;
    if ((s = launch_rows(rp, kv, G, n_sparse + n_win, kv->batch, as_stream(stream), 1, &launched)) != AOH_OK) return s;
    if (launched) return AOH_OK;
  }
  // otherwise the SPARSE heads' step, then the window heads' attention
  if (n_sparse > 0) {
    s = aoh_sparse_decode(q, n_q_heads, kv, idom, n_dom, n_fac, n_fac_per_seq, n_fac_cap, roles, scale, out, idx_out,
                          count_out, workspace, sparse_need, stream);
    if (s != AOH_OK) return s;
  }
  if (n_win > 0)
    return aoh_stream_decode(q, n_q_heads, kv, roles, sink, window, scale, out,
                             static_cast<uint8_t*>(workspace) + sparse_need, win_need, stream);
  return AOH_OK;
}

size_t aoh_shared_index_decode_workspace_size(const aoh_kv_cache* kv, int32_t n_layers, int32_t n_q_heads,
                                              int32_t n_fac_cap) {
  if (check_kv(kv) != AOH_OK || check_heads(kv, n_q_heads) != AOH_OK || n_layers < 1 || n_fac_cap < 1) return 0;
  if (int64_t(n_layers) * (n_q_heads / kv->n_kv_heads) > kMaxQRows) return 0;
  return fd_bytes(shared_geom(kv, n_layers, n_q_heads, n_fac_cap));
}

aoh_status aoh_shared_index_decode(const void* q_layers, int32_t n_layers, int32_t n_q_heads,
                                   const aoh_kv_cache* kv, const int32_t* idx, const int32_t* count,
                                   int32_t n_fac_cap, float scale, float* out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if (is_ring(kv)) return AOH_ERR_INVALID_ARG;  // a ring holds streaming heads only
  if ((s = check_heads(kv, n_q_heads)) != AOH_OK) return s;
  if (n_layers < 1 || n_fac_cap < 1 || !std::isfinite(scale)) return AOH_ERR_INVALID_ARG;
  const int G = n_q_heads / kv->n_kv_heads;
  if (int64_t(n_layers) * G > kMaxQRows) return AOH_ERR_UNSUPPORTED;
  if (kv->batch == 0) return AOH_OK;
  if (!q_layers || !idx || !count || !out) return AOH_ERR_INVALID_ARG;
  if (!aligned16(q_layers)) return AOH_ERR_ALIGNMENT;
  const FdGeom geo = shared_geom(kv, n_layers, n_q_heads, n_fac_cap);
  if (!ws_ok(workspace, workspace_bytes, fd_bytes(geo))) return AOH_ERR_WORKSPACE;
  uint8_t heads[kMaxHeads];
  const int n_listed = list_heads(kv, nullptr, true, heads);
  FdecParams fp{};
  fp.q = static_cast<const uint16_t*>(q_layers);
  fp.k = static_cast<const uint16_t*>(kv->k);
  fp.v = static_cast<const uint16_t*>(kv->v);
  fp.offsets = kv->offsets;
  bind_cache(fp, kv);
  fp.idx = idx;
  fp.count = count;
  fp.out = out;
  fp.stride_tok = kv->stride_tok;
  fp.stride_head = kv->stride_head;
  fp.B = kv->batch;
  fp.Hq = n_q_heads;
  fp.Hkv = kv->n_kv_heads;
  fp.G = G;
  fp.NQ = n_layers * G;
  fp.cap = n_fac_cap;
  fp.list_mode = 1;
  fp.scale_log2 = scale * 1.4426950408889634f;
  memcpy(fp.heads, heads, n_listed);
  fd_bind(fp, geo, static_cast<uint8_t*>(workspace));
  return launch_fd(fp, kv->head_dim, geo.nqp, n_listed, kv->batch, as_stream(stream), true);
}

size_t shared_step_scores_bytes(const aoh_kv_cache* kv) {
  return align256(sizeof(float) * (size_t)kv->n_kv_heads * (size_t)std::max<int64_t>(kv->total_tokens, 1));
}

// [gather partials][scores][select region]
size_t shared_step_ws_bytes(const aoh_kv_cache* kv, int32_t n_layers, int32_t Hq, int32_t topk) {
  return fd_bytes(shared_geom(kv, n_layers, Hq, topk)) + shared_step_scores_bytes(kv) + select_ws(kv).total;
}

size_t aoh_shared_index_step_workspace_size(const aoh_kv_cache* kv, int32_t n_layers, int32_t n_q_heads,
                                            int32_t topk) {
  if (check_kv(kv) != AOH_OK || check_heads(kv, n_q_heads) != AOH_OK || n_layers < 1 || topk < 1) return 0;
  if (int64_t(n_layers) * (n_q_heads / kv->n_kv_heads) > kMaxQRows) return 0;
  return shared_step_ws_bytes(kv, n_layers, n_q_heads, topk);
}

aoh_status aoh_shared_index_step(const void* q_index, const void* q_layers, int32_t n_layers, int32_t n_q_heads,
                                 const aoh_kv_cache* kv, int32_t topk, int32_t* idx, int32_t* count, float scale,
                                 float* out, void* workspace, size_t workspace_bytes, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if (is_ring(kv)) return AOH_ERR_INVALID_ARG;  // a ring holds streaming heads only
  if ((s = check_heads(kv, n_q_heads)) != AOH_OK) return s;
  if (n_layers < 1 || topk < 1 || !std::isfinite(scale)) return AOH_ERR_INVALID_ARG;
  const int G = n_q_heads / kv->n_kv_heads;
  if (int64_t(n_layers) * G > kMaxQRows) return AOH_ERR_UNSUPPORTED;
  if (kv->batch == 0) return AOH_OK;
  if (!q_index || !q_layers || !idx || !count || !out) return AOH_ERR_INVALID_ARG;
  if (!aligned16(q_index) || !aligned16(q_layers)) return AOH_ERR_ALIGNMENT;
  const size_t need = shared_step_ws_bytes(kv, n_layers, n_q_heads, topk);
  if (!ws_ok(workspace, workspace_bytes, need)) return AOH_ERR_WORKSPACE;
  uint8_t heads[kMaxHeads];
  const int n_listed = list_heads(kv, nullptr, true, heads);
  cudaStream_t st = as_stream(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const FdGeom geo = shared_geom(kv, n_layers, n_q_heads, topk);
  float* scores = reinterpret_cast<float*>(ws + fd_bytes(geo));
  if (fused_feasible(kv, n_layers * G)) {
    RowParams rp{};
    rp.q_score = static_cast<const uint16_t*>(q_index);
    rp.q_attn = static_cast<const uint16_t*>(q_layers);
    rp.k = static_cast<const uint16_t*>(kv->k);
    rp.v = static_cast<const uint16_t*>(kv->v);
    rp.offsets = kv->offsets;
    bind_cache(rp, kv);
    rows_score_source(rp, kv, nullptr, kv->head_dim / 2);
    rp.n_fac_per_seq = nullptr;
    rp.n_fac = topk;
    rp.cap = topk;
    rp.idx_out = idx;
    rp.count_out = count;
    rp.out = out;
    rp.stride_tok = kv->stride_tok;
    rp.stride_head = kv->stride_head;
    rp.T = (int32_t)kv->total_tokens;
    rp.B = kv->batch;
    rp.Hq = n_q_heads;
    rp.Hkv = kv->n_kv_heads;
    rp.G = G;
    rp.NQ = n_layers * G;
    rp.scale_log2 = scale * 1.4426950408889634f;
    memcpy(rp.heads, heads, n_listed);
    bool launched = false;
    if ((s = launch_rows(rp, kv, n_layers * G, n_listed, kv->batch, st, 1, &launched)) != AOH_OK) return s;
    if (launched) return AOH_OK;
  }
  // otherwise: full-dimension scores, the select, the shared-index gather
  if (!select_fits(kv)) return AOH_ERR_UNSUPPORTED;
  uint8_t* sel_ws = ws + fd_bytes(geo) + shared_step_scores_bytes(kv);
  if (kv->total_tokens > 0) {
    if ((s = launch_tip_full(q_index, n_q_heads, kv, scores, heads, n_listed, st)) != AOH_OK) return s;
  }
  s = launch_select(scores, kv, topk, nullptr, topk, idx, count, heads, n_listed, sel_ws, st);
  if (s != AOH_OK) return s;
  FdecParams fp{};
  fp.q = static_cast<const uint16_t*>(q_layers);
  fp.k = static_cast<const uint16_t*>(kv->k);
  fp.v = static_cast<const uint16_t*>(kv->v);
  fp.offsets = kv->offsets;
  bind_cache(fp, kv);
  fp.idx = idx;
  fp.count = count;
  fp.out = out;
  fp.stride_tok = kv->stride_tok;
  fp.stride_head = kv->stride_head;
  fp.B = kv->batch;
  fp.Hq = n_q_heads;
  fp.Hkv = kv->n_kv_heads;
  fp.G = G;
  fp.NQ = n_layers * G;
  fp.cap = topk;
  fp.list_mode = 1;
  fp.scale_log2 = scale * 1.4426950408889634f;
  memcpy(fp.heads, heads, n_listed);
  fd_bind(fp, geo, ws);
  return launch_fd(fp, kv->head_dim, geo.nqp, n_listed, kv->batch, st, true);
}

aoh_status aoh_kv_append(const void* q_new, int32_t n_q_heads, const void* k_new, const void* v_new, double theta,
                         const aoh_kv_cache* kv, const aoh_kv_cache* ring, const int32_t* idom, int32_t n_dom,
                         int32_t* lengths, void* q_out, void* stream) {
  if (!kv && !ring) return AOH_ERR_INVALID_ARG;
  aoh_status s;
  if (kv) {
    if ((s = check_kv(kv)) != AOH_OK) return s;
    if (is_ring(kv)) return AOH_ERR_INVALID_ARG;
  }
  if (ring) {
    if ((s = check_kv(ring)) != AOH_OK) return s;
    if (!is_ring(ring)) return AOH_ERR_INVALID_ARG;
    if (ring->k_dom) return AOH_ERR_INVALID_ARG;
  }
  const aoh_kv_cache* any = kv ? kv : ring;
  if (kv && ring && (kv->batch != ring->batch || kv->n_kv_heads != ring->n_kv_heads ||
                     kv->head_dim != ring->head_dim))
    return AOH_ERR_INVALID_ARG;
  for (int g = 0; g < any->n_kv_heads; ++g) {  // every head is kept somewhere
    const bool in_kv = kv && slot_of(kv, g) != kNoSlot, in_ring = ring && slot_of(ring, g) != kNoSlot;
    if (!in_kv && !in_ring) return AOH_ERR_INVALID_ARG;
  }
  if ((q_new == nullptr) != (q_out == nullptr)) return AOH_ERR_INVALID_ARG;
  if (q_new && (n_q_heads < 1 || n_q_heads % any->n_kv_heads)) return AOH_ERR_INVALID_ARG;
  if (!(theta > 0.0) || !std::isfinite(theta)) return AOH_ERR_INVALID_ARG;
  const bool pack = kv && kv->k_dom;
  if (pack && (!idom || n_dom < 1 || n_dom > kv->head_dim / 2 || 2 * n_dom > kv->k_dom_cols))
    return AOH_ERR_INVALID_ARG;
  if (any->batch == 0) return AOH_OK;
  if (!k_new || !v_new || !lengths) return AOH_ERR_INVALID_ARG;
  AppendParams ap{};
  ap.q_new = static_cast<const uint16_t*>(q_new);
  ap.k_new = static_cast<const uint16_t*>(k_new);
  ap.v_new = static_cast<const uint16_t*>(v_new);
  ap.q_out = static_cast<uint16_t*>(q_out);
  ap.lengths = lengths;
  ap.B = any->batch;
  ap.Hq = q_new ? n_q_heads : 0;
  ap.Hkv = any->n_kv_heads;
  ap.d = any->head_dim;
  ap.theta = theta;
  for (int g = 0; g < any->n_kv_heads; ++g) {
    ap.slot[g] = kv ? slot_of(kv, g) : kNoSlot;
    ap.rslot[g] = ring ? slot_of(ring, g) : kNoSlot;
  }
  if (kv) {
    ap.k = static_cast<uint16_t*>(const_cast<void*>(kv->k));
    ap.v = static_cast<uint16_t*>(const_cast<void*>(kv->v));
    ap.offsets = kv->offsets;
    ap.stride_tok = kv->stride_tok;
    ap.stride_head = kv->stride_head;
    ap.T = kv->total_tokens;
    if (pack) {
      ap.k_dom = static_cast<uint16_t*>(const_cast<void*>(kv->k_dom));
      ap.k_dom_cols = kv->k_dom_cols;
      ap.idom = idom;
      ap.n_dom = n_dom;
    }
  }
  if (ring) {
    ap.rk = static_cast<uint16_t*>(const_cast<void*>(ring->k));
    ap.rv = static_cast<uint16_t*>(const_cast<void*>(ring->v));
    ap.roffsets = ring->offsets;
    ap.rstride_tok = ring->stride_tok;
    ap.rstride_head = ring->stride_head;
    ap.ring_sink = ring->ring_sink;
    ap.ring_window = ring->ring_window;
  }
  cudaStream_t st = as_stream(stream);
  before_launch(st);
  kv_append_kernel<<<ap.B, kAppendThreads, 0, st>>>(ap);
  return count_launch(AOH_KERNEL_KV_APPEND, st);
}

}  // extern "C"

// ===================================================================== AoH head classifier
namespace {

struct ClassifyGeom {
  int splits, k_per_split;
  size_t partial_bytes, gram_bytes, work_bytes;
};

// d_model split into CTAs of at most 512 columns (a multiple of 64 that divides d_model)
ClassifyGeom classify_geom(int32_t d_model, int32_t Hq, int32_t Hkv, int32_t D) {
  ClassifyGeom g{};
  int kps = 512;
  while (kps > 64 && d_model % kps) kps -= 64;
  g.k_per_split = kps;
  g.splits = d_model / kps;
  const size_t heads = (size_t)Hq + Hkv, dd = (size_t)D * D;
  g.partial_bytes = align256(heads * g.splits * dd * sizeof(double));
  g.gram_bytes = align256(heads * dd * sizeof(double));
  g.work_bytes = align256((size_t)Hq * dd * sizeof(double));
  return g;
}

aoh_status check_classify(int32_t d_model, int32_t Hq, int32_t Hkv, int32_t D, int32_t n_retrieval) {
  if (D != 64 && D != 128) return AOH_ERR_UNSUPPORTED;
  if (Hkv < 1 || Hkv > kMaxHeads || Hq < 1 || Hq % Hkv) return AOH_ERR_INVALID_ARG;
  if (d_model < D || d_model % 64) return AOH_ERR_INVALID_ARG;
  if (n_retrieval < 0 || n_retrieval > Hkv) return AOH_ERR_INVALID_ARG;
  return AOH_OK;
}

template <int D>
aoh_status launch_classify(const void* w_q, const void* w_k, int32_t d_model, int32_t Hq, int32_t Hkv,
                           int32_t n_retrieval, double* er_heads, double* er_groups, uint8_t* roles, uint8_t* ws,
                           const ClassifyGeom& geo, cudaStream_t st) {
  static std::atomic<uint64_t> configured{0};
  const size_t gram_smem = size_t(kGramStages) * D * kGramPitch * 2;
  const size_t spec_smem = (size_t(D) * (D + 1) + size_t(D) * 8) * sizeof(double);
  if (!set_up_on_this_device(configured)) {
    aoh_status s = set_smem(gram_kernel<D>, gram_smem);
    if (s != AOH_OK) return s;
    if ((s = set_smem(spectrum_kernel<D>, spec_smem)) != AOH_OK) return s;
    mark_set_up(configured);
  }
  double* partial = reinterpret_cast<double*>(ws);
  double* gram = reinterpret_cast<double*>(ws + geo.partial_bytes);
  double* work = reinterpret_cast<double*>(ws + geo.partial_bytes + geo.gram_bytes);
  GramParams gp{};
  gp.wq = static_cast<const uint16_t*>(w_q);
  gp.wk = static_cast<const uint16_t*>(w_k);
  gp.partial = partial;
  gp.d_model = d_model;
  gp.Hq = Hq;
  gp.Hkv = Hkv;
  gp.splits = geo.splits;
  gp.k_per_split = geo.k_per_split;
  before_launch(st);
  gram_kernel<D><<<dim3(geo.splits, Hq + Hkv, 2), kGramThreads, gram_smem, st>>>(gp);
  aoh_status s = count_launch(AOH_KERNEL_GRAM, st);
  if (s != AOH_OK) return s;
  const int64_t n = int64_t(Hq + Hkv) * D * D;
  before_launch(st);
  gram_reduce_kernel<<<(unsigned)std::min<int64_t>(ceil_div(n, 256), int64_t(sm_count()) * 8), 256, 0, st>>>(
      partial, gram, Hq + Hkv, geo.splits, D * D);
  if ((s = count_launch(AOH_KERNEL_GRAM_REDUCE, st)) != AOH_OK) return s;
  SpectrumParams sp{};
  sp.gram = gram;
  sp.work = work;
  sp.er_heads = er_heads;
  sp.Hq = Hq;
  sp.Hkv = Hkv;
  sp.G = Hq / Hkv;
  before_launch(st);
  spectrum_kernel<D><<<Hq, kSpecThreads, spec_smem, st>>>(sp);
  if ((s = count_launch(AOH_KERNEL_SPECTRUM, st)) != AOH_OK) return s;
  RolesParams rp{};
  rp.er_heads = er_heads;
  rp.er_groups = er_groups;
  rp.roles = roles;
  rp.Hkv = Hkv;
  rp.G = Hq / Hkv;
  rp.n_retrieval = n_retrieval;
  before_launch(st);
  group_roles_kernel<<<1, 128, 0, st>>>(rp);
  return count_launch(AOH_KERNEL_GROUP_ROLES, st);
}

}  // namespace

extern "C" size_t aoh_head_classify_workspace_size(int32_t d_model, int32_t n_q_heads, int32_t n_kv_heads,
                                                  int32_t head_dim) {
  if (check_classify(d_model, n_q_heads, n_kv_heads, head_dim, 0) != AOH_OK) return 0;
  const ClassifyGeom g = classify_geom(d_model, n_q_heads, n_kv_heads, head_dim);
  return g.partial_bytes + g.gram_bytes + g.work_bytes;
}

extern "C" aoh_status aoh_head_classify(const void* w_q, const void* w_k, int32_t d_model, int32_t n_q_heads,
                                        int32_t n_kv_heads, int32_t head_dim, int32_t n_retrieval, double* er_heads,
                                        double* er_groups, uint8_t* roles, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  aoh_status s = check_classify(d_model, n_q_heads, n_kv_heads, head_dim, n_retrieval);
  if (s != AOH_OK) return s;
  if (!w_q || !w_k || !er_heads || !er_groups || !roles) return AOH_ERR_INVALID_ARG;
  if (!aligned16(w_q) || !aligned16(w_k)) return AOH_ERR_ALIGNMENT;
  const ClassifyGeom geo = classify_geom(d_model, n_q_heads, n_kv_heads, head_dim);
  if (!ws_ok(workspace, workspace_bytes, geo.partial_bytes + geo.gram_bytes + geo.work_bytes)) return AOH_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (head_dim == 128)
    return launch_classify<128>(w_q, w_k, d_model, n_q_heads, n_kv_heads, n_retrieval, er_heads, er_groups, roles, ws,
                                geo, as_stream(stream));
  return launch_classify<64>(w_q, w_k, d_model, n_q_heads, n_kv_heads, n_retrieval, er_heads, er_groups, roles, ws,
                             geo, as_stream(stream));
}

// ===================================================================== FASA-M host offload
namespace {

// The device-side address of a buffer the GPU can reach (device memory, or pinned host memory
// mapped into the device's address space); pageable host memory is refused.
aoh_status device_view(const void* p, const void** out) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return AOH_ERR_INVALID_ARG;
  }
  if (a.type == cudaMemoryTypeUnregistered || a.devicePointer == nullptr) return AOH_ERR_INVALID_ARG;
  *out = a.devicePointer;
  return AOH_OK;
}

aoh_status check_offload(const aoh_offload_cache* oc, int32_t n_dom) {
  if (!oc) return AOH_ERR_INVALID_ARG;
  if (oc->batch < 0 || oc->n_kv_heads < 1 || oc->n_kv_heads > kMaxHeads) return AOH_ERR_INVALID_ARG;
  if (oc->head_dim != 64 && oc->head_dim != 128) return AOH_ERR_UNSUPPORTED;
  if (oc->max_len < 0 || oc->total_tokens < 0 || oc->total_tokens >= (int64_t(1) << 31)) return AOH_ERR_INVALID_ARG;
  if (n_dom < 1 || n_dom > oc->head_dim / 2) return AOH_ERR_INVALID_ARG;
  if (n_dom % 4) return AOH_ERR_UNSUPPORTED;  // the dominant part of a row is whole 16-byte segments
  if (oc->k_dom_cols < 2 * n_dom || oc->k_dom_cols > 128 || oc->k_dom_cols % 8) return AOH_ERR_INVALID_ARG;
  if (oc->rest_cols < oc->head_dim - 2 * n_dom || oc->rest_cols % 8 || oc->rest_cols > oc->head_dim)
    return AOH_ERR_INVALID_ARG;
  if (oc->batch == 0) return AOH_OK;
  if (!oc->offsets || !oc->k_dom || !oc->k_rest || !oc->v) return AOH_ERR_INVALID_ARG;
  if (!aligned16(oc->k_dom) || !aligned16(oc->k_rest) || !aligned16(oc->v)) return AOH_ERR_ALIGNMENT;
  return AOH_OK;
}

// A cache descriptor over the device part only (the packed dominant columns): what the scan
// and the select read.  Its k / v point at k_dom as well but are never read.
aoh_kv_cache offload_device_part(const aoh_offload_cache* oc) {
  aoh_kv_cache kv{};
  kv.k = kv.v = oc->k_dom;
  kv.offsets = oc->offsets;
  kv.lengths = oc->lengths;
  kv.batch = oc->batch;
  kv.n_kv_heads = oc->n_kv_heads;
  kv.head_dim = oc->head_dim;
  kv.max_len = oc->max_len;
  kv.total_tokens = oc->total_tokens;
  kv.stride_tok = oc->k_dom_cols;
  kv.stride_head = std::max<int64_t>(oc->total_tokens, 1) * oc->k_dom_cols;
  kv.k_dom = oc->k_dom;
  kv.k_dom_cols = oc->k_dom_cols;
  return kv;
}

struct OffloadWs {
  size_t fd, scores, idx, count, sidx, soff, sk, sv, sq, sel, total;
};

OffloadWs offload_ws(const aoh_offload_cache* oc, int32_t Hq, int32_t cap) {
  const aoh_kv_cache kv = offload_device_part(oc);
  OffloadWs w{};
  const size_t B = (size_t)oc->batch, H = (size_t)oc->n_kv_heads, d = (size_t)oc->head_dim;
  size_t o = 0;
  w.fd = o;
  o += fd_bytes(sparse_geom(&kv, Hq, cap));
  w.scores = o;
  o += align256(sizeof(float) * H * (size_t)std::max<int64_t>(oc->total_tokens, 1));
  w.idx = o;
  o += align256(sizeof(int32_t) * B * H * cap);
  w.count = o;
  o += align256(sizeof(int32_t) * B * H);
  w.sidx = o;
  o += align256(sizeof(int32_t) * B * H * cap);
  w.soff = o;
  o += align256(sizeof(int32_t) * (B + 1));
  w.sk = o;
  o += align256(2 * B * cap * H * d);
  w.sv = o;
  o += align256(2 * B * cap * H * d);
  w.sq = o;
  o += align256(2 * B * (size_t)Hq * d);
  w.sel = o;
  o += select_ws(&kv).total;
  w.total = o;
  return w;
}

}  // namespace

extern "C" aoh_status aoh_offload_split(const aoh_kv_cache* kv, const int32_t* idom, int32_t n_dom, void* k_rest,
                                        int32_t rest_cols, void* v_host, void* stream) {
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if (is_ring(kv)) return AOH_ERR_INVALID_ARG;
  if (n_dom < 1 || n_dom > kv->head_dim / 2) return AOH_ERR_INVALID_ARG;
  if (n_dom % 4) return AOH_ERR_UNSUPPORTED;
  if (rest_cols < kv->head_dim - 2 * n_dom || rest_cols % 8 || rest_cols > kv->head_dim) return AOH_ERR_INVALID_ARG;
  for (int g = 0; g < kv->n_kv_heads; ++g)
    if (slot_of(kv, g) == kNoSlot) return AOH_ERR_INVALID_ARG;  // every head is split
  if (kv->batch == 0 || kv->total_tokens == 0) return AOH_OK;
  if (!idom || !k_rest || !v_host) return AOH_ERR_INVALID_ARG;
  if (!aligned16(k_rest) || !aligned16(v_host)) return AOH_ERR_ALIGNMENT;
  const void *kr = nullptr, *vh = nullptr;
  if ((s = device_view(k_rest, &kr)) != AOH_OK) return s;
  if ((s = device_view(v_host, &vh)) != AOH_OK) return s;
  SplitParams sp{};
  sp.k = static_cast<const uint16_t*>(kv->k);
  sp.v = static_cast<const uint16_t*>(kv->v);
  sp.stride_tok = kv->stride_tok;
  sp.stride_head = kv->stride_head;
  sp.idom = idom;
  sp.k_rest = static_cast<uint16_t*>(const_cast<void*>(kr));
  sp.v_host = static_cast<uint16_t*>(const_cast<void*>(vh));
  sp.T = (int32_t)kv->total_tokens;
  sp.d = kv->head_dim;
  sp.n_dom = n_dom;
  sp.rest_cols = rest_cols;
  for (int g = 0; g < kv->n_kv_heads; ++g) sp.slot[g] = slot_of(kv, g);
  const int slabs = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(kv->total_tokens, 64),
                                                                 ceil_div(int64_t(sm_count()) * 4, kv->n_kv_heads)));
  cudaStream_t st = as_stream(stream);
  before_launch(st);
  offload_split_kernel<<<dim3(slabs, kv->n_kv_heads), kStageThreads, 0, st>>>(sp);
  return count_launch(AOH_KERNEL_OFFLOAD_SPLIT, st);
}

extern "C" size_t aoh_offload_decode_workspace_size(const aoh_offload_cache* oc, int32_t n_q_heads,
                                                   int32_t n_fac_cap) {
  if (!oc || oc->n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % oc->n_kv_heads || n_fac_cap < 1) return 0;
  if (oc->head_dim != 64 && oc->head_dim != 128) return 0;
  if (n_q_heads / oc->n_kv_heads > kMaxQRows) return 0;
  return offload_ws(oc, n_q_heads, n_fac_cap).total;
}

extern "C" aoh_status aoh_offload_decode(const void* q, int32_t n_q_heads, const aoh_offload_cache* oc,
                                         const int32_t* idom, int32_t n_dom, int32_t n_fac,
                                         const int32_t* n_fac_per_seq, int32_t n_fac_cap, float scale, float* out,
                                         int32_t* idx_out, int32_t* count_out, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  aoh_status s = check_offload(oc, n_dom);
  if (s != AOH_OK) return s;
  if (n_q_heads < 1 || n_q_heads % oc->n_kv_heads) return AOH_ERR_INVALID_ARG;
  const int G = n_q_heads / oc->n_kv_heads;
  if (G > kMaxQRows) return AOH_ERR_UNSUPPORTED;
  if (n_fac_cap < 1 || (!n_fac_per_seq && (n_fac < 0 || n_fac > n_fac_cap))) return AOH_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return AOH_ERR_INVALID_ARG;
  if ((idx_out == nullptr) != (count_out == nullptr)) return AOH_ERR_INVALID_ARG;
  if (oc->batch == 0) return AOH_OK;
  if (!q || !idom || !out) return AOH_ERR_INVALID_ARG;
  if (!aligned16(q)) return AOH_ERR_ALIGNMENT;
  const OffloadWs wl = offload_ws(oc, n_q_heads, n_fac_cap);
  if (!ws_ok(workspace, workspace_bytes, wl.total)) return AOH_ERR_WORKSPACE;
  const void *kr = nullptr, *vh = nullptr;
  if ((s = device_view(oc->k_rest, &kr)) != AOH_OK) return s;
  if ((s = device_view(oc->v, &vh)) != AOH_OK) return s;
  const aoh_kv_cache kv = offload_device_part(oc);
  uint8_t heads[kMaxHeads];
  const int Hkv = oc->n_kv_heads, d = oc->head_dim;
  for (int g = 0; g < Hkv; ++g) heads[g] = (uint8_t)g;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* scores = reinterpret_cast<float*>(ws + wl.scores);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + wl.idx);
  int32_t* cnt = count_out ? count_out : reinterpret_cast<int32_t*>(ws + wl.count);
  cudaStream_t st = as_stream(stream);
  // 1-2. importance scan of the dominant columns (on the GPU) and the top-N_fac select
  if (!select_fits(&kv)) return AOH_ERR_UNSUPPORTED;
  if (kv.total_tokens > 0 && (s = launch_tip(q, n_q_heads, &kv, idom, n_dom, scores, heads, Hkv, st)) != AOH_OK)
    return s;
  if ((s = launch_select(scores, &kv, n_fac, n_fac_per_seq, n_fac_cap, idx, cnt, heads, Hkv, ws + wl.sel, st)) !=
      AOH_OK)
    return s;
  // 3. the selected rows across the host link, into HBM
  StageParams sp{};
  sp.q = static_cast<const uint16_t*>(q);
  sp.k_dom = static_cast<const uint16_t*>(oc->k_dom);
  sp.k_rest = static_cast<const uint16_t*>(kr);
  sp.v_host = static_cast<const uint16_t*>(vh);
  sp.idom = idom;
  sp.offsets = oc->offsets;
  sp.lengths = oc->lengths;
  sp.idx = idx;
  sp.count = cnt;
  sp.sk = reinterpret_cast<uint16_t*>(ws + wl.sk);
  sp.sv = reinterpret_cast<uint16_t*>(ws + wl.sv);
  sp.sq = reinterpret_cast<uint16_t*>(ws + wl.sq);
  sp.sidx = reinterpret_cast<int32_t*>(ws + wl.sidx);
  sp.soffsets = reinterpret_cast<int32_t*>(ws + wl.soff);
  sp.T = oc->total_tokens;
  sp.B = oc->batch;
  sp.Hq = n_q_heads;
  sp.Hkv = Hkv;
  sp.G = G;
  sp.d = d;
  sp.n_dom = n_dom;
  sp.k_dom_cols = oc->k_dom_cols;
  sp.rest_cols = oc->rest_cols;
  sp.cap = n_fac_cap;
  memcpy(sp.heads, heads, Hkv);
  before_launch(st);
  offload_stage_kernel<<<dim3(Hkv, oc->batch), kStageThreads, 0, st>>>(sp);
  if ((s = count_launch(AOH_KERNEL_OFFLOAD_STAGE, st)) != AOH_OK) return s;
  // 4. focused attention over the staged rows (identity index, dominant-first dim order)
  const FdGeom geo = sparse_geom(&kv, n_q_heads, n_fac_cap);
  FdecParams fp{};
  fp.q = sp.sq;
  fp.k = sp.sk;
  fp.v = sp.sv;
  fp.offsets = sp.soffsets;
  fp.lengths = nullptr;
  fp.idx = sp.sidx;
  fp.count = cnt;
  fp.out = out;
  fp.stride_tok = int64_t(Hkv) * d;
  fp.stride_head = d;
  fp.B = oc->batch;
  fp.Hq = n_q_heads;
  fp.Hkv = Hkv;
  fp.G = G;
  fp.NQ = G;
  fp.cap = n_fac_cap;
  fp.list_mode = 1;
  fp.scale_log2 = scale * 1.4426950408889634f;
  memcpy(fp.heads, heads, Hkv);
  for (int g = 0; g < Hkv; ++g) fp.slot[g] = (uint8_t)g;
  fd_bind(fp, geo, ws + wl.fd);
  return launch_fd(fp, d, geo.nqp, Hkv, oc->batch, st, n_fac_per_seq == nullptr);
}

// ===================================================================== no-allocation variant
// Scratch for aoh_stream_decode_noalloc: a file-scope device array, so the call needs no
// allocation.  Every device that loads the library holds it until the process exits.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
std::mutex g_static_mu;
void* g_static_addr[256];  // device address of the array last set up, per device ordinal (host-side)

// The array's device address on the current device, looked up on every call (a host-side
// query, no synchronisation), so that a context created after cudaDeviceReset, which loads
// the module again, is never handed a stale address.  When the address is new for this
// device the array is zeroed (the split counters at its head must start at zero; every
// later call leaves them at zero) and the device synchronised: the first call on a device,
// and the first after a reset, must therefore not happen during a stream capture.
aoh_status static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaGetLastError());
  if (dev < 0 || dev >= 256) return AOH_ERR_UNSUPPORTED;
  void* ptr = nullptr;
  aoh_status s = cuda_status(cudaGetSymbolAddress(&ptr, g_static_scratch));
  if (s != AOH_OK) return s;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_addr[dev] != ptr) {
    if ((s = cuda_status(cudaMemset(ptr, 0, kStaticScratchBytes))) != AOH_OK) return s;
    if ((s = cuda_status(cudaDeviceSynchronize())) != AOH_OK) return s;
    g_static_addr[dev] = ptr;
  }
  *out = ptr;
  return AOH_OK;
}
}  // namespace

extern "C" aoh_status aoh_stream_decode_noalloc(const void* q, int32_t n_q_heads, const aoh_kv_cache* kv,
                                                const uint8_t* roles, int32_t sink, int32_t window, float scale,
                                                float* out, void* stream) {
  // every argument check of aoh_stream_decode runs before the scratch is touched
  aoh_status s = check_kv(kv);
  if (s != AOH_OK) return s;
  if ((s = check_heads(kv, n_q_heads)) != AOH_OK) return s;
  if (!roles) return AOH_ERR_INVALID_ARG;
  if ((s = check_roles(kv, roles)) != AOH_OK) return s;
  if (n_q_heads / kv->n_kv_heads > kMaxQRows) return AOH_ERR_UNSUPPORTED;
  if (sink < 0 || window < 0 || !std::isfinite(scale)) return AOH_ERR_INVALID_ARG;
  if ((s = check_ring_roles(kv, roles, sink, window)) != AOH_OK) return s;
  if (kv->batch == 0) return AOH_OK;
  if (!q || !out) return AOH_ERR_INVALID_ARG;
  if (!aligned16(q)) return AOH_ERR_ALIGNMENT;
  if (fd_bytes(stream_geom(kv, n_q_heads, roles, sink, window)) > kStaticScratchBytes) return AOH_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = static_scratch_address(&scratch)) != AOH_OK) return s;
  return aoh_stream_decode(q, n_q_heads, kv, roles, sink, window, scale, out, scratch, kStaticScratchBytes, stream);
}
