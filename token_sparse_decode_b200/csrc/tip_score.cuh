// Token Importance Predictor scan (FASA: Frequency-aware Sparse Attention, §2.B.1).
// (Rows are addressed through each KV head's slot in the cache; the unused tail of a
// sequence's region, when the cache carries per-sequence lengths, is not scored.)
//
// For KV head g of sequence b the score of cached token t is the fp32 dot of
//   q~_g = sum over the group's q heads of q_h, restricted to the dominant dims
//          {c, c + d/2 : c in I_dom[g]} (zero elsewhere)
// with the key row.  By linearity this is the per-head chunk sum of the method
// aggregated over the GQA group.  The kernel is a persistent streaming GEMV: every
// CTA streams an equal share of the (head, token) rows, every key row is read once
// with 16-byte vector loads, S = row_bytes/16 lanes share a row and reduce with
// shuffles.  Two row sources:
//   packed   k_dom[g][t][0 .. cols)  (dominant columns only: 4*n_dom bytes a row)
//   in place K[t][g][0 .. d)         (16-byte segments holding no dominant dim
//                                     are not loaded)
#pragma once

#include "device_common.cuh"

namespace aoh {

constexpr int kTipThreads = 256;

struct TipParams {
  const uint16_t* q;        // [B][Hq][d]
  const uint16_t* src;      // packed k_dom or K
  const int32_t* idom;      // [Hkv][n_dom]; null: every chunk (K in place)
  const int32_t* offsets;   // [B + 1]
  const int32_t* lengths;   // [B] or null (sequences fill their regions)
  float* scores;            // [Hkv][T]
  int64_t row_stride_tok;   // elements between token rows of one head
  int64_t row_stride_head;  // elements between heads
  int32_t T, Hq, Hkv, d, G, n_dom;
  int32_t row_len;          // elements per row: k_dom cols (packed) or d (in place)
  int32_t packed;
  int32_t B;
  int64_t per_cta;          // flattened (listed head, token) rows per CTA
  int64_t total;            // n_listed * T
  uint8_t heads[kMaxHeads]; // KV heads scored
  uint8_t slot[kMaxHeads];  // head slot of every KV head in the row source
};

// S = lanes per row: row_len / 8 rounded up to a power of two (1 .. 16); lanes whose
// 16-byte segment lies past the row end carry zero weights and load nothing.
//
// Persistent grid: CTA c owns rows [c * per_cta, (c + 1) * per_cta) of the flattened
// (listed head j, token t) space, so every CTA streams the same number of rows.  A CTA walks
// its share segment by segment (a segment = the rows of one head within one sequence); at a
// segment start it issues the first batch of row loads, then finds the sequence and builds
// q~ while those loads are in flight.
template <int S>
__global__ void __launch_bounds__(kTipThreads, 4) tip_score_kernel(const TipParams p) {
  grid_dep_launch();  // the select that follows may begin scheduling
  __shared__ float qt[128];
  __shared__ int s_seg[3];  // sequence b of the segment (-1: none), its region's end, its last token + 1
  const int tid = threadIdx.x, lane = tid & 31;
  const int C = p.d >> 1;
  const int seg = lane % S;
  constexpr int RPI = kTipThreads / S;  // rows per block iteration
  constexpr int U = 8;                  // independent loads in flight per thread
  constexpr int BATCH = U * RPI;
  const int prow = (tid >> 5) * (32 / S) + lane / S;
  const int64_t w1 = min(p.total, (int64_t)(blockIdx.x + 1) * p.per_cta);
  int64_t w = (int64_t)blockIdx.x * p.per_cta;
  int bhint = 0;
  int64_t cur_j = -1;
  while (w < w1) {  // CTA-uniform
    const int64_t j = w / p.T;
    const int t = (int)(w - j * p.T);
    const int g = p.heads[j];
    const int lim = (int)min(w1 - w, (j + 1) * (int64_t)p.T - w);  // rows of this head in the share
    // the rows' segment columns: in place with I_dom, segments without a dominant dim stay unread
    bool active = true;
    if (!p.packed && p.idom) {
      active = false;
      for (int jj = 0; jj < p.n_dom; ++jj) {
        const int c = p.idom[g * p.n_dom + jj];
        const int lo = seg * 8, hi = seg * 8 + 8;
        if ((c >= lo && c < hi) || (c + C >= lo && c + C < hi)) active = true;
      }
    }
    active = active && seg * 8 < p.row_len;
    const uint16_t* base = p.src + (int64_t)p.slot[g] * p.row_stride_head + (int64_t)t * p.row_stride_tok + seg * 8;
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = u * RPI + prow;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (r < lim && active) v[u] = ld_stream_v4(base + (int64_t)r * p.row_stride_tok);
    }
    // the segment: sequence b holding token t (searched from the previous one within a head)
    if (j != cur_j) bhint = 0;
    cur_j = j;
    if (tid < 32) {
      int b = -1;
      for (int b0 = bhint; b0 < p.B && b < 0; b0 += 32) {
        const int i = b0 + lane;
        const bool hit = i < p.B && p.offsets[i] <= t && t < p.offsets[i + 1];
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) b = b0 + __ffs(m) - 1;
      }
      if (lane == 0) {
        int e = p.T, ve = p.T;
        if (b < 0) {
          record_error(kCheckPosition, (int)j, t, -1);
        } else {
          e = p.offsets[b + 1];
          if (e > p.T) {  // offsets past the cache: score no row beyond it
            record_error(kCheckPosition, (int)j, e, p.T);
            e = p.T;
          }
          int off;
          ve = p.lengths ? min(e, p.offsets[b] + seq_length(p.offsets, p.lengths, b, false, &off)) : e;
        }
        s_seg[0] = b;
        s_seg[1] = e;
        s_seg[2] = ve;
      }
    }
    __syncthreads();
    const int b = s_seg[0];
    if (t >= s_seg[2]) {  // the unused tail of a sequence's region: nothing to score
      w += min(lim, s_seg[1] - t);
      __syncthreads();    // s_seg is rewritten by the next segment
      continue;
    }
    const int n = min(lim, s_seg[2] - t);  // rows of the segment (>= 1)
    if (b >= 0) bhint = b;
    // q~ for (b, g): fp32 group sum in head order, restricted to the dominant dims
    if (tid < p.row_len) {
      int dim = -1;
      if (b < 0) {
      } else if (p.packed) {
        if (tid < 2 * p.n_dom) {
          const int jj = tid < p.n_dom ? tid : tid - p.n_dom;
          const int c = p.idom[g * p.n_dom + jj];
          if (c < 0 || c >= C) {
            record_error(kCheckChunk, g, jj, c);
          } else {
            dim = tid < p.n_dom ? c : c + C;
          }
        }
      } else if (p.idom == nullptr) {
        dim = tid;  // every chunk: the full dot
      } else {
        const int c = tid < C ? tid : tid - C;
        for (int jj = 0; jj < p.n_dom; ++jj) {
          const int cj = p.idom[g * p.n_dom + jj];
          if (cj < 0 || cj >= C) record_error(kCheckChunk, g, jj, cj);
          if (cj == c) dim = tid;
        }
      }
      float acc = 0.f;
      if (dim >= 0) {
        const uint16_t* qb = p.q + ((int64_t)b * p.Hq + (int64_t)g * p.G) * p.d + dim;
        for (int h = 0; h < p.G; ++h) acc += __uint_as_float((uint32_t)qb[(int64_t)h * p.d] << 16);
      }
      qt[tid] = acc;
    }
    __syncthreads();
    float qs[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) qs[i] = (seg * 8 + i < p.row_len) ? qt[seg * 8 + i] : 0.f;
    __syncthreads();  // qt is rewritten by the next segment
    float* srow = p.scores + (int64_t)g * p.T + t;
    for (int r0 = 0; r0 < n; r0 += BATCH) {  // CTA-uniform trip count: full-mask shuffles
      if (r0 > 0) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int r = r0 + u * RPI + prow;
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (r < n && active) v[u] = ld_stream_v4(base + (int64_t)r * p.row_stride_tok);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float sc = dot8(v[u], qs);
#pragma unroll
        for (int o = S / 2; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
        const int r = r0 + u * RPI + prow;
        if (seg == 0 && r < n) srow[r] = sc;
      }
    }
    w += n;
  }
}

// ------------------------------------------------------------------ dominant-column packing
struct PackParams {
  const uint16_t* k;
  const int32_t* idom;
  uint16_t* k_dom;          // [head slots][T][cols]
  int64_t stride_tok, stride_head;
  int32_t T, n_listed, d, n_dom, cols;
  uint8_t heads[kMaxHeads]; // KV heads the cache stores
  uint8_t slot[kMaxHeads];  // their head slots (in K and in k_dom)
};

__global__ void __launch_bounds__(256) pack_dominant_kernel(const PackParams p) {
  const int C = p.d >> 1;
  const int64_t n_rows = (int64_t)p.n_listed * p.T;
  const int64_t total = n_rows * p.cols;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(e % p.cols);
    const int64_t row = e / p.cols;
    const int g = p.heads[row / p.T];
    const int s = p.slot[g];
    const int64_t t = row % p.T;
    uint16_t val = 0;
    if (j < 2 * p.n_dom) {
      const int c = p.idom[g * p.n_dom + (j < p.n_dom ? j : j - p.n_dom)];
      if (c < 0 || c >= C) {
        record_error(kCheckChunk, g, j, c);
      } else {
        const int dim = j < p.n_dom ? c : c + C;
        val = p.k[t * p.stride_tok + (int64_t)s * p.stride_head + dim];
      }
    }
    p.k_dom[((int64_t)s * p.T + t) * p.cols + j] = val;
  }
}

}  // namespace aoh
