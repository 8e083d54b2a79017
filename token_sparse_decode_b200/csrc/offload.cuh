// FASA-M: the cache split between GPU and host memory (FASA: Frequency-aware Sparse
// Attention, §2.C: the value cache and the non-dominant parts of the keys go to CPU
// memory; only the dominant components stay on the GPU).
//
// Layouts (head-major, token t of head g):
//   device  k_dom  [Hkv][T][k_dom_cols]: dims I_dom, then I_dom + d/2 (as packed for the scan)
//   host    k_rest [Hkv][T][rest_cols]:  the other d - 2 n_dom dims in ascending order
//   host    v      [Hkv][T][d]
// Host arrays are pinned and mapped: kernels read and write them over the host link.
//
// A decode step scans k_dom and selects on the GPU like the resident path; then
// offload_stage_kernel brings only the selected rows across the link into HBM: the K row
// reassembled in the head's dominant-first dim order [I_dom, I_dom + d/2, rest] and the V
// row as it is, plus the group's q rows permuted the same way (q.k is a sum over dims, so
// it is unchanged by a permutation applied to both).  Focused attention then runs on the
// staged rows with the identity index.  Per selected token and head the link carries
// 2 * (rest_cols + d) bytes.
#pragma once

#include "device_common.cuh"

namespace aoh {

constexpr int kStageThreads = 256;
constexpr int kStageU = 8;  // 16-byte loads in flight per thread

// rest[i] = the i-th dim outside the dominant chunks of head g (ascending), i < d - 2 n_dom;
// perm[i] = the dominant-first order [I_dom, I_dom + d/2, rest].  Called by every thread.
// (I_dom entries must be distinct chunk ids in [0, d/2); an entry outside that range is
// recorded as check 3 and perm then stays a permutation of some dims, never past d.)
__device__ __forceinline__ void head_dim_order(const int32_t* idom_g, int n_dom, int d, uint8_t* perm,
                                               int* s_scan) {
  const int C = d >> 1, tid = threadIdx.x;
  if (tid < d) perm[tid] = (uint8_t)tid;
  if (tid < n_dom && (idom_g[tid] < 0 || idom_g[tid] >= C)) record_error(kCheckChunk, tid, idom_g[tid], C);
  bool dom = false;
  if (tid < d) {
    const int c = tid < C ? tid : tid - C;
    for (int j = 0; j < n_dom; ++j) dom |= (idom_g[j] == c);
  }
  int total;
  const int rank = block_exclusive_scan((tid < d && !dom) ? 1 : 0, s_scan, &total);  // ends with a barrier
  if (tid < d) {
    if (dom) {
      const int c = tid < C ? tid : tid - C;
      int j = 0;
      while (j < n_dom && idom_g[j] != c) ++j;
      perm[tid < C ? j : n_dom + j] = (uint8_t)tid;
    } else if (2 * n_dom + rank < d) {
      perm[2 * n_dom + rank] = (uint8_t)tid;
    }
  }
  __syncthreads();
}

struct SplitParams {
  const uint16_t* k;          // device cache K (strided, head slots)
  const uint16_t* v;
  int64_t stride_tok, stride_head;
  const int32_t* idom;        // [Hkv][n_dom]
  uint16_t* k_rest;           // host [Hkv][T][rest_cols]
  uint16_t* v_host;           // host [Hkv][T][d]
  int32_t T, d, n_dom, rest_cols;
  uint8_t slot[kMaxHeads];
};

// One CTA per (KV head, slab of tokens): writes the head's host rows, one 16-byte store per
// 8 elements (each store crosses the host link).
__global__ void __launch_bounds__(kStageThreads) offload_split_kernel(const SplitParams p) {
  __shared__ uint8_t perm[128];
  __shared__ int s_scan[33];
  const int g = blockIdx.y;
  head_dim_order(p.idom + g * p.n_dom, p.n_dom, p.d, perm, s_scan);
  const int nrest = p.d - 2 * p.n_dom;
  const int64_t per = (p.T + gridDim.x - 1) / gridDim.x;
  const int64_t t0 = blockIdx.x * per, t1 = min((int64_t)p.T, t0 + per);
  const int rc = p.rest_cols / 8, vc = p.d / 8;  // 16-byte chunks of a rest row and of a value row
  const int64_t row_chunks = rc + vc;
  for (int64_t e = t0 * row_chunks + threadIdx.x; e < t1 * row_chunks; e += kStageThreads) {
    const int64_t t = e / row_chunks;
    const int c = (int)(e % row_chunks);
    const uint16_t* kr = p.k + t * p.stride_tok + (int64_t)p.slot[g] * p.stride_head;
    const uint16_t* vr = p.v + t * p.stride_tok + (int64_t)p.slot[g] * p.stride_head;
    if (c < rc) {
      uint16_t x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = c * 8 + u;
        x[u] = i < nrest ? kr[perm[2 * p.n_dom + i]] : (uint16_t)0;
      }
      uint4 w;
      w.x = (uint32_t)x[0] | ((uint32_t)x[1] << 16);
      w.y = (uint32_t)x[2] | ((uint32_t)x[3] << 16);
      w.z = (uint32_t)x[4] | ((uint32_t)x[5] << 16);
      w.w = (uint32_t)x[6] | ((uint32_t)x[7] << 16);
      *reinterpret_cast<uint4*>(p.k_rest + ((int64_t)g * p.T + t) * p.rest_cols + c * 8) = w;
    } else {
      const int j = c - rc;
      *reinterpret_cast<uint4*>(p.v_host + ((int64_t)g * p.T + t) * p.d + j * 8) =
          *reinterpret_cast<const uint4*>(vr + j * 8);
    }
  }
}

struct StageParams {
  const uint16_t* q;          // [B][Hq][d]
  const uint16_t* k_dom;      // device [Hkv][T][k_dom_cols]
  const uint16_t* k_rest;     // host [Hkv][T][rest_cols]
  const uint16_t* v_host;     // host [Hkv][T][d]
  const int32_t* idom;
  const int32_t* offsets;     // [B + 1] of the cache
  const int32_t* lengths;     // [B] or null
  const int32_t* idx;         // [B][Hkv][cap] the selection
  const int32_t* count;       // [B][Hkv]
  uint16_t* sk;               // staged K [B * cap][Hkv][d] (dominant-first order)
  uint16_t* sv;               // staged V [B * cap][Hkv][d]
  uint16_t* sq;               // staged q [B][Hq][d] (dominant-first order per group)
  int32_t* sidx;              // [B][Hkv][cap]: the identity list
  int32_t* soffsets;          // [B + 1]: b * cap
  int64_t T;
  int32_t B, Hq, Hkv, G, d, n_dom, k_dom_cols, rest_cols, cap;
  uint8_t heads[kMaxHeads];
};

// One CTA per (listed KV head, sequence): the selected rows of that row of the index.
__global__ void __launch_bounds__(kStageThreads) offload_stage_kernel(const StageParams p) {
  __shared__ uint8_t perm[128];
  __shared__ int s_scan[33];
  __shared__ int s_pos[1024];
  const int b = blockIdx.y, g = p.heads[blockIdx.x], tid = threadIdx.x;
  head_dim_order(p.idom + g * p.n_dom, p.n_dom, p.d, perm, s_scan);
  if (blockIdx.x == 0 && b == 0)
    for (int i = tid; i <= p.B; i += kStageThreads) p.soffsets[i] = i * p.cap;
  // the group's q rows in the head's order
  for (int e = tid; e < p.G * p.d; e += kStageThreads) {
    const int hh = g * p.G + e / p.d, i = e % p.d;
    p.sq[((int64_t)b * p.Hq + hh) * p.d + i] = p.q[((int64_t)b * p.Hq + hh) * p.d + perm[i]];
  }
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  int n = p.count[b * p.Hkv + g];
  if (n > p.cap || n < 0) {
    if (tid == 0) record_error(kCheckCount, b, g, n);
    n = n < 0 ? 0 : p.cap;
  }
  int32_t* sidx = p.sidx + ((int64_t)b * p.Hkv + g) * p.cap;
  for (int j = tid; j < p.cap; j += kStageThreads) sidx[j] = j < n ? j : -1;
  const int32_t* lst = p.idx + ((int64_t)b * p.Hkv + g) * p.cap;
  const int dom_chunks = (2 * p.n_dom) / 8, row_chunks = p.d / 8;
  const int per_tok = 2 * row_chunks;  // K chunks, then V chunks
  for (int j0 = 0; j0 < n; j0 += 1024) {
    const int nj = min(1024, n - j0);
    __syncthreads();
    for (int j = tid; j < nj; j += kStageThreads) {
      int pos = lst[j0 + j];
      if (pos < 0 || pos >= L) {
        record_error(kCheckPosition, b, g, pos);
        pos = -1;
      }
      s_pos[j] = pos;
    }
    __syncthreads();
    const int items = nj * per_tok;
    for (int e0 = tid; e0 < items; e0 += kStageThreads * kStageU) {
      uint4 val[kStageU];
#pragma unroll
      for (int u = 0; u < kStageU; ++u) {  // every load issued before any store
        const int e = e0 + u * kStageThreads;
        val[u] = make_uint4(0u, 0u, 0u, 0u);
        if (e < items) {
          const int j = e / per_tok, c = e % per_tok;
          const int pos = s_pos[j];
          if (pos >= 0) {
            const int64_t t = (int64_t)off + pos;
            const uint16_t* src;
            if (c < dom_chunks)
              src = p.k_dom + ((int64_t)g * p.T + t) * p.k_dom_cols + c * 8;
            else if (c < row_chunks)
              src = p.k_rest + ((int64_t)g * p.T + t) * p.rest_cols + (c - dom_chunks) * 8;
            else
              src = p.v_host + ((int64_t)g * p.T + t) * p.d + (c - row_chunks) * 8;
            val[u] = *reinterpret_cast<const uint4*>(src);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kStageU; ++u) {
        const int e = e0 + u * kStageThreads;
        if (e < items) {
          const int j = e / per_tok, c = e % per_tok;
          const int64_t row = ((int64_t)b * p.cap + j0 + j) * p.Hkv + g;
          uint16_t* dst = c < row_chunks ? p.sk + row * p.d + c * 8 : p.sv + row * p.d + (c - row_chunks) * 8;
          *reinterpret_cast<uint4*>(dst) = val[u];
        }
      }
    }
  }
}

}  // namespace aoh
