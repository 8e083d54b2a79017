// Gather flash-decode: exact softmax attention of NQ query rows over a list of
// cached token positions of one KV head.
//
// Serves three operations with one body:
//   * focused attention over the selected tokens (FASA: Frequency-aware Sparse
//     Attention, §2.B.2): positions come from the top-N_fac index, NQ = G;
//   * retrieval / streaming heads (AoH summary, Metodología §4): positions are
//     [0, L) or [0, min(S, L)) U [max(S, L - W), L), NQ = G; a streaming head may
//     keep its rows in a ring of sink + window slots (then position p is read
//     from slot ring_slot(p));
//   * the shared-index cross-decoder layers ("Cómo funciona CLSA"): one index,
//     NQ = n_layers * G query rows read every gathered K/V row once.
//
// Work split: blockIdx = (split, listed KV head, sequence).  A CTA owns `chunk`
// consecutive list entries, streams their K and V rows through a 3-stage cp.async
// pipeline into 128-byte-swizzled shared tiles, and runs the contraction on tensor cores
// with the tokens on the M side:
//     S^T[16 tok x 8 q] = K[16 tok x d] . Q^T[d x 8 q]          (m16n8k16, bf16)
//     O^T[d x 8 q]     += V^T[d x 16 tok] . P^T[16 tok x 8 q]
// so G <= 8 query rows fill the N = 8 side of one MMA (G = 7: 7/8 useful) instead
// of padding 16 rows.  NT n-tiles of 8 query rows, each with 4 (NT <= 2) or 2
// (NT = 4) warps over the stage's 16-token sub-tiles.  P goes from the accumulator
// layout to the B-operand layout with movmatrix.trans.  Softmax is online in fp32
// (exp2 domain).  Each CTA leaves (m, l, acc) for its chunk; they are merged either
// in a thread-block cluster of the row's splits (rows of about equal length with
// 2-16 splits: distributed shared memory, each CTA writes 1/CL of the outputs, every
// thread fetching its row's (m, l) and the peers' partials in one round of remote loads
// per 8 peers) or by the last CTA of the row through the workspace (atomic ticket,
// re-armed to zero).
#pragma once

#include <cooperative_groups.h>

#include "device_common.cuh"

namespace aoh {

// token-group warps for every n-tile of 8 query rows: 4 (one or two n-tiles) or 2 (four n-tiles),
// so a CTA has 128 or 256 threads and two fit an SM
__host__ __device__ constexpr int fd_groups(int nt) { return nt == 4 ? 2 : 4; }
__host__ __device__ constexpr int fd_threads(int nt) { return 32 * nt * fd_groups(nt); }
constexpr int kFdTS = 64;        // tokens per pipeline stage
constexpr int kFdStages = 3;
constexpr bool kFdWarpRing = true;  // role ranges, up to 8 query rows: warp-private rings (no block barrier per stage)
constexpr int kFdPosCap = 1024;  // list positions staged in shared memory per CTA
constexpr int kFdMaxSplits = 256; // splits per row (the combine stages their weights in shared memory)
constexpr int kFdMaxCluster = 16;  // splits of a row merged through distributed shared memory
// cluster merge buffers start past the warps' partials [warps][8][2 + D] floats
__host__ __device__ constexpr int fd_merge_off(int nt, int d) { return ((nt * fd_groups(nt) * 8 * (2 + d) * 4) + 255) & ~255; }

struct FdecParams {
  const uint16_t* q;         // row (layer l, b, h) at q + ((l * B + b) * Hq + h) * D
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* offsets;    // [B + 1]
  const int32_t* lengths;    // [B] or null (sequences fill their regions)
  const int32_t* idx;        // list mode: [B][Hkv][cap]
  const int32_t* count;      // list mode: [B][Hkv]
  float* out;                // row (l, b, h) at out + ((l * B + b) * Hq + h) * D
  float* part_ml;            // [rows][max_splits][NQP][2]
  float* part_acc;           // [rows][max_splits][NQP][D]
  int32_t* tickets;          // [rows], zero between calls
  int64_t stride_tok, stride_head;
  int32_t B, Hq, Hkv, G, NQ, cap;
  int32_t chunk;             // list entries per CTA, multiple of kFdTS
  int32_t max_splits;
  int32_t list_mode;         // 1: positions from idx/count; 0: role ranges
  int32_t cluster_combine;   // 1: launched with clusters of max_splits CTAs (one row each)
  int32_t defer_merge;       // 1: the CTAs of a row with several splits only leave their partials
                             //    (flash_merge_kernel combines them)
  int32_t q_split;           // CTAs sharing a row's positions, each with NQP of its query rows (0 or 1:
                             //    one); blockIdx.y = listed head * q_split + part
  int32_t sink, window;
  int32_t ring_sink, ring_window;  // range mode on a ring cache (> 0 sum): position p is kept in
                                   // slot ring_slot(p); 0, 0: position p is token p of the region
  float scale_log2;          // softmax scale * log2(e)
  uint8_t heads[kMaxHeads];  // listed KV heads (blockIdx.y)
  uint8_t roles[kMaxHeads];  // role of every KV head (range mode)
  uint8_t slot[kMaxHeads];   // head slot of every KV head in K / V
};

template <int D>
struct FdTile {
  static constexpr int kTileBytes = kFdTS * D * 2;      // one of K or V per stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kSmem = kFdStages * kStageBytes;
};

// Byte offset of (row r, dim dd) in a [kFdTS x D] bf16 tile stored as D/64 column
// halves of [kFdTS x 128 B], 16-byte chunks XOR-swizzled by (r mod 8).
__device__ __forceinline__ uint32_t fd_tile_off(int r, int dd) {
  const int half = dd >> 6;
  const int cc = (dd & 63) >> 3;
  return (uint32_t)(half * (kFdTS * 128) + r * 128 + ((cc ^ (r & 7)) << 4));
}

// The number of positions row (b, g) attends to, and for a role range the split [0, ra) U
// [rb, L): list mode takes the selection's count (clamped to [0, cap]); a ring region too small
// for its slots attends to nothing.
__device__ __forceinline__ int fd_row_count(const FdecParams& p, int b, int g, int L, int off, bool ring, int* ra,
                                            int* rb) {
  *ra = 0;
  *rb = 0;
  if (p.list_mode) return max(0, min(p.count[b * p.Hkv + g], p.cap));
  if (ring && p.offsets[b + 1] - off < p.ring_sink + p.ring_window) return 0;
  if (p.roles[g] == 1) {  // DENSE
    *ra = L;
    *rb = L;
  } else {                // STREAM
    *ra = min(p.sink, L);
    *rb = max(*ra, L - p.window);
  }
  return *ra + (L - *rb);
}

// The end of a gather CTA, shared by both gather kernels: red_ml [NT * WT][8][2] and red_acc
// [NT * WT][8][D] (floats at the start of the dynamic shared memory) hold the partial (m, l, acc)
// of each (n-tile nt, token group t) at index nt + NT * t; the groups are merged, then the
// row's splits (cluster merge, the row's last CTA through the workspace, or partials left for
// flash_merge_kernel).  MERGE_OFF: where the cluster merge buffers start.
template <int D, int NT, int WT, int THREADS, int MERGE_OFF>
__device__ __forceinline__ void fd_finish(const FdecParams& p, uint8_t* smem, int* s_last_p, int tid, int b, int g,
                                          int q0, int nq, int row_id, int split, int nsplit, bool clus) {
  constexpr int kFdThreads = THREADS;
  constexpr int kFdMergeOff = MERGE_OFF;
  constexpr int NQP = NT * 8;
  constexpr int NW = NT * WT;
  int& s_last = *s_last_p;
  const float* red_ml = reinterpret_cast<const float*>(smem);  // [NW][8][2]
  const float* red_acc = red_ml + NW * 8 * 2;                  // [NW][8][D]
  if (clus) {
    // ---- cluster merge: every CTA leaves (M, L, A) of its split in shared memory (past the
    // warp partials), then CTA r combines outputs r, r + CL, ... over the CL splits
    namespace cgs = cooperative_groups;
    cgs::cluster_group cluster = cgs::this_cluster();
    const int CLn = (int)cluster.num_blocks(), rk = (int)cluster.block_rank();
    float* cm = reinterpret_cast<float*>(smem + kFdMergeOff);  // [NQP]
    float* cls = cm + NQP;                                      // [NQP]
    float* ca = cls + NQP;                                      // [NQP][D]
    for (int e = tid; e < NQP * D; e += kFdThreads) {
      const int qr = e / D, dd = e % D;
      const int ntq = qr >> 3, cq = qr & 7;
      float M = -INFINITY;
#pragma unroll
      for (int t = 0; t < WT; ++t) M = fmaxf(M, red_ml[((ntq + NT * t) * 8 + cq) * 2]);
      float Ls = 0.f, A = 0.f;
#pragma unroll
      for (int t = 0; t < WT; ++t) {
        const int w = ntq + NT * t;
        const float mw = red_ml[(w * 8 + cq) * 2];
        const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
        Ls += f * red_ml[(w * 8 + cq) * 2 + 1];
        A += f * red_acc[(w * 8 + cq) * D + dd];
      }
      ca[e] = A;
      if (dd == 0) {
        cm[qr] = M;
        cls[qr] = Ls;
      }
    }
    cluster.sync();
    // outputs 4 consecutive dims at a time: each thread fetches its row's (M, L) from every
    // peer together with the peers' 16-byte partials (batches of 8 peers, all of a batch's
    // remote loads in flight together; a running rescale joins the batches)
    for (int e4 = rk * kFdThreads + tid; e4 < nq * D / 4; e4 += CLn * kFdThreads) {
      const int e = 4 * e4, qr = e / D, dd = e % D;
      float Mx = -INFINITY, Ls = 0.f;
      float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int pq = 0; pq < CLn; pq += 8) {
        float mv[8], lv[8];
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (pq + u < CLn) {
            mv[u] = cluster.map_shared_rank(cm, pq + u)[qr];
            lv[u] = cluster.map_shared_rank(cls, pq + u)[qr];
            v[u] = *reinterpret_cast<const float4*>(cluster.map_shared_rank(ca, pq + u) + e);
          } else {
            mv[u] = -INFINITY;
            lv[u] = 0.f;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float Mb = Mx;
#pragma unroll
        for (int u = 0; u < 8; ++u) Mb = fmaxf(Mb, mv[u]);
        const float sc = (Mx == -INFINITY) ? 0.f : exp2f(Mx - Mb);
        Ls *= sc;
        A.x *= sc;
        A.y *= sc;
        A.z *= sc;
        A.w *= sc;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float w = (mv[u] == -INFINITY) ? 0.f : exp2f(mv[u] - Mb);
          Ls += w * lv[u];
          A.x += w * v[u].x;
          A.y += w * v[u].y;
          A.z += w * v[u].z;
          A.w += w * v[u].w;
        }
        Mx = Mb;
      }
      const float inv = 1.f / Ls;
      const int l = (q0 + qr) / p.G, h = g * p.G + (q0 + qr) % p.G;
      float* o = p.out + (((int64_t)l * p.B + b) * p.Hq + h) * D + dd;
      o[0] = A.x * inv;
      o[1] = A.y * inv;
      o[2] = A.z * inv;
      o[3] = A.w * inv;
    }
    cluster.sync();  // peers read this CTA's shared memory until here
    return;
  }
  const bool single = (nsplit == 1);
  float* pml = p.part_ml + ((int64_t)row_id * p.max_splits + split) * NQP * 2;
  float* pacc = p.part_acc + ((int64_t)row_id * p.max_splits + split) * NQP * D;
  for (int e = tid; e < NQP * D; e += kFdThreads) {
    const int qr = e / D, dd = e % D;
    const int ntq = qr >> 3, cq = qr & 7;
    float M = -INFINITY;
#pragma unroll
    for (int t = 0; t < WT; ++t) M = fmaxf(M, red_ml[((ntq + NT * t) * 8 + cq) * 2]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int t = 0; t < WT; ++t) {
      const int w = ntq + NT * t;
      const float mw = red_ml[(w * 8 + cq) * 2];
      const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
      Ls += f * red_ml[(w * 8 + cq) * 2 + 1];
      A += f * red_acc[(w * 8 + cq) * D + dd];
    }
    if (single) {
      if (qr < nq) {
        const int l = (q0 + qr) / p.G, h = g * p.G + (q0 + qr) % p.G;
        p.out[(((int64_t)l * p.B + b) * p.Hq + h) * D + dd] = A / Ls;
      }
    } else {
      pacc[qr * D + dd] = A;
      if (dd == 0) {
        pml[qr * 2] = M;
        pml[qr * 2 + 1] = Ls;
      }
    }
  }
  if (single || p.defer_merge) return;

  // ---- split-K combine by the last CTA of the row
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int ticket = atomicAdd(p.tickets + row_id, 1);
    s_last = (ticket == nsplit - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* rml = p.part_ml + (int64_t)row_id * p.max_splits * NQP * 2;
  const float* racc = p.part_acc + (int64_t)row_id * p.max_splits * NQP * D;
  // weights w[s][q] = 2^(m_sq - M_q) staged in shared memory (nsplit * NQP <= kFdMaxSplits * NQP fits).
  // The partials sit in L2: the max and sum run over all threads, the weighted sum keeps 16
  // independent loads in flight per thread.
  float* sw = reinterpret_cast<float*>(smem);        // [nsplit][NQP]
  float* sM = sw + nsplit * NQP;                     // [NQP]
  float* sL = sM + NQP;                              // [NQP]
  float* sred = sL + NQP;                            // [kFdThreads]: per-thread partial max / sum
  // every thread takes query row tid % NQP over the splits j, j + SP, ... (SP = threads / NQP)
  constexpr int SP = kFdThreads / NQP;
  const int rq = tid % NQP, sj = tid / NQP;
  {
    float M = -INFINITY;
    for (int s2 = sj; s2 < nsplit; s2 += SP) M = fmaxf(M, __ldcg(rml + ((int64_t)s2 * NQP + rq) * 2));
    sred[tid] = M;
  }
  __syncthreads();
  if (tid < NQP) {
    float M = -INFINITY;
    for (int j = 0; j < SP; ++j) M = fmaxf(M, sred[j * NQP + tid]);
    sM[tid] = M;
  }
  __syncthreads();
  for (int e = tid; e < nsplit * NQP; e += kFdThreads) {
    const int qr = e % NQP;
    sw[e] = exp2f(__ldcg(rml + (int64_t)e * 2) - sM[qr]);
  }
  __syncthreads();
  {
    float Ls = 0.f;
    for (int s2 = sj; s2 < nsplit; s2 += SP) Ls += sw[s2 * NQP + rq] * __ldcg(rml + ((int64_t)s2 * NQP + rq) * 2 + 1);
    sred[tid] = Ls;
  }
  __syncthreads();
  if (tid < NQP) {
    float Ls = 0.f;
    for (int j = 0; j < SP; ++j) Ls += sred[j * NQP + tid];
    sL[tid] = Ls;
  }
  __syncthreads();
  // four consecutive dimensions of one query row per thread
  for (int e4 = tid; e4 < nq * (D / 4); e4 += kFdThreads) {
    const int qr = e4 / (D / 4), dd = (e4 % (D / 4)) * 4;
    const float* col = racc + (int64_t)qr * D + dd;
    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
    int s2 = 0;
    for (; s2 + 16 <= nsplit; s2 += 16) {
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = __ldcg(reinterpret_cast<const float4*>(col + (int64_t)(s2 + u) * NQP * D));
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float w = sw[(s2 + u) * NQP + qr];
        A.x += w * v[u].x;
        A.y += w * v[u].y;
        A.z += w * v[u].z;
        A.w += w * v[u].w;
      }
    }
    for (; s2 < nsplit; ++s2) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(col + (int64_t)s2 * NQP * D));
      const float w = sw[s2 * NQP + qr];
      A.x += w * v.x;
      A.y += w * v.y;
      A.z += w * v.z;
      A.w += w * v.w;
    }
    const float inv = 1.f / sL[qr];
    const int l = (q0 + qr) / p.G, h = g * p.G + (q0 + qr) % p.G;
    float* o = p.out + (((int64_t)l * p.B + b) * p.Hq + h) * D + dd;
    o[0] = A.x * inv;
    o[1] = A.y * inv;
    o[2] = A.z * inv;
    o[3] = A.w * inv;
  }
  if (tid == 0) p.tickets[row_id] = 0;
}

template <int D, int NT>
__global__ void __launch_bounds__(fd_threads(NT)) flash_gather_kernel(const FdecParams p) {
  constexpr int ST = kFdStages;
  grid_dep_wait();  // the selection comes from the kernel before this one
  grid_dep_launch();
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(NT == 1 || NT == 2 || NT == 4, "n-tiles");
  constexpr int KS = D / 16;         // k-steps of QK, m-tiles of PV
  constexpr int WT = fd_groups(NT);  // token groups (warps sharing one n-tile)
  constexpr int kFdThreads = fd_threads(NT);
  constexpr int NW = kFdThreads / 32;
  constexpr int kFdMergeOff = fd_merge_off(NT, D);
  constexpr int SUB = kFdTS / 16;    // 16-token sub-tiles per stage
  constexpr int NQP = NT * 8;        // padded query rows
  constexpr int CPR = D / 8;         // 16-byte chunks per row
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ int s_last;
  __shared__ int s_pos[kFdPosCap];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.z;
  const int y = blockIdx.y;
  const int QS = max(1, p.q_split);
  const int g = p.heads[y / QS];
  const int q0 = (y % QS) * NQP;               // this CTA's first query row
  const int nq = max(0, min(NQP, p.NQ - q0));  // and its number of query rows
  const int split = blockIdx.x;
  const int row_id = b * gridDim.y + y;
  const bool ring = (p.ring_sink + p.ring_window) > 0;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, ring, &off);

  // ---- the row's list of positions
  int ra, rb;
  const int n = fd_row_count(p, b, g, L, off, ring, &ra, &rb);
  if (p.list_mode && split == 0 && tid == 0 && p.count[b * p.Hkv + g] > p.cap)
    record_error(kCheckCount, b, g, p.count[b * p.Hkv + g]);
  const int32_t* lst = p.list_mode ? p.idx + ((int64_t)b * p.Hkv + g) * p.cap : nullptr;
  const int nsplit = (n + p.chunk - 1) / p.chunk;

  if (n == 0) {  // nothing to attend to: zero rows
    if (ring && split == 0 && tid == 0 && p.offsets[b + 1] - off < p.ring_sink + p.ring_window)
      record_error(kCheckCapacity, b, p.offsets[b + 1] - off, p.ring_sink + p.ring_window);
    if (split == 0) {
      for (int e = tid; e < nq * D; e += kFdThreads) {
        const int qr = q0 + e / D, l = qr / p.G, h = g * p.G + qr % p.G;
        p.out[(((int64_t)l * p.B + b) * p.Hq + h) * D + e % D] = 0.f;
      }
    }
    return;
  }
  const bool clus = p.cluster_combine != 0;
  if (split >= nsplit && !clus) return;  // in a cluster an idle split still takes part in the merge
  const int j0 = split * p.chunk;
  const int ntok = max(0, min(n, j0 + p.chunk) - j0);
  const int nstages = (ntok + kFdTS - 1) / kFdTS;

  // list mode: stage this CTA's positions once (one round trip instead of one per stage)
  const bool pos_in_smem = p.list_mode && ntok <= kFdPosCap;
  if (pos_in_smem) {
    for (int j = tid; j < ntok; j += kFdThreads) {
      int pos = __ldg(lst + j0 + j);
      if (pos < 0 || pos >= L) {
        record_error(kCheckPosition, b, g, pos);
        pos = -1;
      }
      s_pos[j] = pos;
    }
    __syncthreads();
  }

  const uint16_t* kbase = p.k + (int64_t)off * p.stride_tok + (int64_t)p.slot[g] * p.stride_head;
  const uint16_t* vbase = p.v + (int64_t)off * p.stride_tok + (int64_t)p.slot[g] * p.stride_head;
  const uint32_t sbase = smem_u32(smem);

  auto issue_stage = [&](int st) {
    if (st < nstages) {
      const uint32_t kt = sbase + (st % ST) * FdTile<D>::kStageBytes;
      const uint32_t vt = kt + FdTile<D>::kTileBytes;
#pragma unroll
      for (int c = tid; c < kFdTS * CPR; c += kFdThreads) {
        const int r = c / CPR, ch = c % CPR;
        const int jj = st * kFdTS + r;  // entry within this CTA's chunk
        bool ok = jj < ntok;
        int pos = 0;
        if (ok) {
          const int j = j0 + jj;
          if (pos_in_smem) {
            pos = s_pos[jj];
            if (pos < 0) {
              ok = false;
              pos = 0;
            }
          } else if (p.list_mode) {
            pos = __ldg(lst + j);
            if (pos < 0 || pos >= L) {
              if (ch == 0) record_error(kCheckPosition, b, g, pos);
              ok = false;
              pos = 0;
            }
          } else {
            pos = j < ra ? j : rb + (j - ra);
            if (ring) pos = ring_slot(pos, p.ring_sink, p.ring_window);
          }
        }
        const int64_t eo = (int64_t)pos * p.stride_tok + ch * 8;
        const uint32_t so = fd_tile_off(r, ch * 8);
        cp_async_16(kt + so, kbase + eo, ok);
        cp_async_16(vt + so, vbase + eo, ok);
      }
    }
    cp_async_commit();
  };

  // ---- Q as B fragments: column n = lane/4 of the warp's n-tile
  const int nt = warp % NT, tg = warp / NT;
  uint32_t bq[KS][2];
  {
    const int qr = nt * 8 + (lane >> 2);
    if (qr < nq) {
      const int l = (q0 + qr) / p.G, h = g * p.G + (q0 + qr) % p.G;
      const uint16_t* qp = p.q + (((int64_t)l * p.B + b) * p.Hq + h) * D + 2 * (lane & 3);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        bq[ks][0] = *reinterpret_cast<const uint32_t*>(qp + ks * 16);
        bq[ks][1] = *reinterpret_cast<const uint32_t*>(qp + ks * 16 + 8);
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) bq[ks][0] = bq[ks][1] = 0u;
    }
  }

  float acc[KS][4];
#pragma unroll
  for (int i = 0; i < KS; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // q rows 2*(lane%4) and +1

  // (row r, dim dd) of a tile of `rows` rows stored as D/64 column halves of [rows x 128 B],
  // 16-byte chunks XOR-swizzled by (r mod 8) (fd_tile_off for rows = kFdTS)
  auto tile_off = [](int rows, int r, int dd) -> uint32_t {
    const int half = dd >> 6;
    const int cc = (dd & 63) >> 3;
    return (uint32_t)(half * (rows * 128) + r * 128 + ((cc ^ (r & 7)) << 4));
  };
  // one 16-token sub-tile: rows r0 .. r0 + 15 of the K / V tiles at kt / vt, nv >= 1 of them valid
  auto sub_tile = [&](uint32_t kt, uint32_t vt, int rows, int r0, int nv) {
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int r = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int dsel = (lane >> 4) * 8;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, kt + tile_off(rows, r, ks * 16 + dsel));
        mma_16816(s4, a, bq[ks][0], bq[ks][1]);
      }
    }
    const int ta = lane >> 2, tb = ta + 8;
    const float x0 = ta < nv ? s4[0] * p.scale_log2 : -INFINITY;
    const float x1 = ta < nv ? s4[1] * p.scale_log2 : -INFINITY;
    const float x2 = tb < nv ? s4[2] * p.scale_log2 : -INFINITY;
    const float x3 = tb < nv ? s4[3] * p.scale_log2 : -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: nv >= 1
    const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
    const float p0 = exp2f(x0 - mn0), p1 = exp2f(x1 - mn1);
    const float p2 = exp2f(x2 - mn0), p3 = exp2f(x3 - mn1);
    l0 = l0 * al0 + p0 + p2;
    l1 = l1 * al1 + p1 + p3;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int i2 = 0; i2 < KS; ++i2) {
      acc[i2][0] *= al0;
      acc[i2][1] *= al1;
      acc[i2][2] *= al0;
      acc[i2][3] *= al1;
    }
    // P enters the PV product as hi + lo bf16 parts (p = hi + lo to ~2^-17), so the
    // weights are not rounded to 8 bits: with few tokens that rounding alone reaches 2e-3.
    const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
    const uint32_t l01 = pack_bf16x2(p0 - bf16lo(h01), p1 - bf16hi(h01));
    const uint32_t l23 = pack_bf16x2(p2 - bf16lo(h23), p3 - bf16hi(h23));
    const uint32_t pb0 = movmatrix_trans(h01), pb1 = movmatrix_trans(h23);
    const uint32_t pl0 = movmatrix_trans(l01), pl1 = movmatrix_trans(l23);
    {
      const int r = r0 + (lane & 7) + (lane >> 4) * 8;
      const int dsel = ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        uint32_t a[4];
        ldsm_x4_trans(a, vt + tile_off(rows, r, mt * 16 + dsel));
        mma_16816(acc[mt], a, pb0, pb1);
        mma_16816(acc[mt], a, pl0, pl1);
      }
    }
  };

  if (NT == 1 && kFdWarpRing && !p.list_mode) {
    // Warp-private rings (role ranges, up to 8 query rows): warp tg owns the sub-tiles u = tg,
    // tg + WT, ... of the chunk (16 tokens each; the same split as the block ring), copies their
    // K / V rows itself into its own ring of ST slots and waits only for its own copies (a warp
    // barrier, no block barrier): a warp goes on as soon as its rows have landed instead of
    // waiting for the slowest copy of the stage.  Measured faster on the contiguous role ranges
    // and not on scattered selections, which keep the block ring.
    constexpr int kSubBytes = 16 * D * 2;  // one 16-row tile of K or V
    const uint32_t wbase = sbase + warp * (ST * 2 * kSubBytes);
    const int nsub = (ntok + 15) / 16;
    const int my_n = nsub > tg ? (nsub - tg + WT - 1) / WT : 0;
    auto issue_w = [&](int k) {
      if (k < my_n) {
        const int u = tg + WT * k;
        const uint32_t kt = wbase + (k % ST) * 2 * kSubBytes;
        const uint32_t vt = kt + kSubBytes;
#pragma unroll
        for (int c = lane; c < 16 * CPR; c += 32) {
          const int r = c / CPR, ch = c % CPR;
          const int jj = u * 16 + r;  // entry within this CTA's chunk
          bool ok = jj < ntok;
          int pos = 0;
          if (ok) {
            const int j = j0 + jj;
            if (pos_in_smem) {
              pos = s_pos[jj];
              if (pos < 0) {
                ok = false;
                pos = 0;
              }
            } else if (p.list_mode) {
              pos = __ldg(lst + j);
              if (pos < 0 || pos >= L) {
                if (ch == 0) record_error(kCheckPosition, b, g, pos);
                ok = false;
                pos = 0;
              }
            } else {
              pos = j < ra ? j : rb + (j - ra);
              if (ring) pos = ring_slot(pos, p.ring_sink, p.ring_window);
            }
          }
          const int64_t eo = (int64_t)pos * p.stride_tok + ch * 8;
          const uint32_t so = tile_off(16, r, ch * 8);
          cp_async_16(kt + so, kbase + eo, ok);
          cp_async_16(vt + so, vbase + eo, ok);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int k = 0; k < ST - 1; ++k) issue_w(k);
    for (int k = 0; k < my_n; ++k) {
      issue_w(k + ST - 1);     // into the slot this warp read at k - 1
      cp_async_wait<ST - 1>();  // this lane's copies of sub-tile k have landed
      __syncwarp();             // and so have the other lanes' (the tile mixes them)
      const int u = tg + WT * k;
      const uint32_t kt = wbase + (k % ST) * 2 * kSubBytes;
      sub_tile(kt, kt + kSubBytes, 16, 0, ntok - u * 16);
      __syncwarp();             // every lane is done with the slot before it is refilled
    }
  } else {
#pragma unroll
    for (int s = 0; s < ST - 1; ++s) issue_stage(s);

    for (int st = 0; st < nstages; ++st) {
      cp_async_wait<ST - 2>();
      __syncthreads();
      issue_stage(st + ST - 1);
      const uint32_t kt = sbase + (st % ST) * FdTile<D>::kStageBytes;
      const uint32_t vt = kt + FdTile<D>::kTileBytes;
#pragma unroll
      for (int i = 0; i < SUB / WT; ++i) {
        const int u = tg + WT * i;
        const int nv = ntok - (st * kFdTS + u * 16);  // valid tokens in this sub-tile
        if (nv <= 0) break;                           // warp-uniform
        sub_tile(kt, vt, kFdTS, u * 16, nv);
      }
    }
  }
  cp_async_wait<0>();

  // ---- merge the WT token groups of every n-tile, through shared memory
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __syncthreads();  // every warp is done with the stage buffers
  float* red_ml = reinterpret_cast<float*>(smem);             // [NW warps][8][2]
  float* red_acc = red_ml + NW * 8 * 2;                       // [NW warps][8][D]
  {
    const int c0 = 2 * (lane & 3);
    if (lane < 4) {
      red_ml[(warp * 8 + c0) * 2 + 0] = m0;
      red_ml[(warp * 8 + c0) * 2 + 1] = l0;
      red_ml[(warp * 8 + c0 + 1) * 2 + 0] = m1;
      red_ml[(warp * 8 + c0 + 1) * 2 + 1] = l1;
    }
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
      const int d0 = mt * 16 + (lane >> 2);
      red_acc[(warp * 8 + c0) * D + d0] = acc[mt][0];
      red_acc[(warp * 8 + c0 + 1) * D + d0] = acc[mt][1];
      red_acc[(warp * 8 + c0) * D + d0 + 8] = acc[mt][2];
      red_acc[(warp * 8 + c0 + 1) * D + d0 + 8] = acc[mt][3];
    }
  }
  __syncthreads();

  fd_finish<D, NT, WT, kFdThreads, kFdMergeOff>(p, smem, &s_last, tid, b, g, q0, nq, row_id, split, nsplit, clus);
}

// Split-K combine of rows with many splits, spread over CTAs: grid (slices of 16 float4
// outputs, listed heads, sequences), 128 threads.  Every CTA stages the row's (m, l) pairs in
// shared memory and weighs the splits itself (w[s][q] = 2^(m_sq - M_q), L_q = sum of w l, in
// split order), then thread (o, s0) sums splits s0, s0 + 8, ...
// of output float4 o with all of its loads in flight, and the 8 split groups are added in a
// fixed order.  Rows with one split were written by the gather.
constexpr int kFmThreads = 128;
constexpr int kFmOut = 16;                    // float4 outputs per CTA
constexpr int kFmGroups = kFmThreads / kFmOut;  // 8 split groups

template <int D, int NT>
__global__ void __launch_bounds__(kFmThreads) flash_merge_kernel(const FdecParams p) {
  grid_dep_wait();  // the partials come from the gather before this launch
  constexpr int NQP = NT * 8;
  extern __shared__ __align__(16) uint8_t fm_smem[];
  float* sml = reinterpret_cast<float*>(fm_smem);  // [nsplit][NQP][2]: (m, l), then (w, l)
  __shared__ float sL[NQP];
  __shared__ float4 sred[kFmGroups][kFmOut];
  const int tid = threadIdx.x;
  const int QS = max(1, p.q_split);
  const int b = blockIdx.z, y = blockIdx.y, g = p.heads[y / QS];
  const int q0 = (y % QS) * NQP, nq = max(0, min(NQP, p.NQ - q0));
  const int row_id = b * gridDim.y + y;
  const bool ring = (p.ring_sink + p.ring_window) > 0;
  int off, ra, rb;
  const int L = seq_length(p.offsets, p.lengths, b, ring, &off);
  const int n = fd_row_count(p, b, g, L, off, ring, &ra, &rb);
  const int nsplit = (n + p.chunk - 1) / p.chunk;
  const int n_out = nq * (D / 4);
  const int o0 = blockIdx.x * kFmOut;
  if (nsplit <= 1 || o0 >= n_out) return;
  const float* rml = p.part_ml + (int64_t)row_id * p.max_splits * NQP * 2;
  const float* racc = p.part_acc + (int64_t)row_id * p.max_splits * NQP * D;
  // weights: the row's (m, l) pairs staged in shared memory with one pass of independent
  // loads, then per query row M_q = max m, w[s][q] = 2^(m_sq - M_q), L_q = sum of w l
  for (int e = tid; e < nsplit * NQP * 2; e += kFmThreads) sml[e] = __ldcg(rml + e);
  __syncthreads();
  // thread t takes query row t % NQP over the splits t / NQP, + SP, ...; the partial maxima
  // and sums are combined in a fixed order
  constexpr int SP = kFmThreads / NQP;
  __shared__ float s_part[kFmThreads], sM[NQP];
  const int rq = tid % NQP, sj = tid / NQP;
  {
    float M = -INFINITY;
    for (int s2 = sj; s2 < nsplit; s2 += SP) M = fmaxf(M, sml[(s2 * NQP + rq) * 2]);
    s_part[tid] = M;
  }
  __syncthreads();
  if (tid < NQP) {
    float M = -INFINITY;
    for (int j2 = 0; j2 < SP; ++j2) M = fmaxf(M, s_part[j2 * NQP + tid]);
    sM[tid] = M;
  }
  __syncthreads();
  {
    float Ls = 0.f;
    for (int s2 = sj; s2 < nsplit; s2 += SP) {
      const float m = sml[(s2 * NQP + rq) * 2];
      const float w = (m == -INFINITY) ? 0.f : exp2f(m - sM[rq]);
      sml[(s2 * NQP + rq) * 2] = w;  // the weight replaces m
      Ls += w * sml[(s2 * NQP + rq) * 2 + 1];
    }
    s_part[tid] = Ls;
  }
  __syncthreads();
  if (tid < NQP) {
    float Ls = 0.f;
    for (int j2 = 0; j2 < SP; ++j2) Ls += s_part[j2 * NQP + tid];
    sL[tid] = Ls;
  }
  __syncthreads();
  // the weighted sums
  const int ol = tid % kFmOut, s0 = tid / kFmOut;
  const int o = o0 + ol;
  float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
  if (o < n_out) {
    const int qr = o / (D / 4), dd = (o % (D / 4)) * 4;
    const float* col = racc + (int64_t)qr * D + dd;
    for (int sb = s0; sb < nsplit; sb += kFmGroups * 16) {
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int s2 = sb + u * kFmGroups;
        v[u] = s2 < nsplit ? __ldcg(reinterpret_cast<const float4*>(col + (int64_t)s2 * NQP * D))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int s2 = sb + u * kFmGroups;
        const float w = s2 < nsplit ? sml[(s2 * NQP + qr) * 2] : 0.f;
        A.x += w * v[u].x;
        A.y += w * v[u].y;
        A.z += w * v[u].z;
        A.w += w * v[u].w;
      }
    }
  }
  sred[s0][ol] = A;
  __syncthreads();
  if (s0 == 0 && o < n_out) {
    float4 T = sred[0][ol];
#pragma unroll
    for (int j = 1; j < kFmGroups; ++j) {
      T.x += sred[j][ol].x;
      T.y += sred[j][ol].y;
      T.z += sred[j][ol].z;
      T.w += sred[j][ol].w;
    }
    const int qr = o / (D / 4), dd = (o % (D / 4)) * 4;
    const float inv = 1.f / sL[qr];
    const int l = (q0 + qr) / p.G, h = g * p.G + (q0 + qr) % p.G;
    float* out = p.out + (((int64_t)l * p.B + b) * p.Hq + h) * D + dd;
    out[0] = T.x * inv;
    out[1] = T.y * inv;
    out[2] = T.z * inv;
    out[3] = T.w * inv;
  }
}

}  // namespace aoh
