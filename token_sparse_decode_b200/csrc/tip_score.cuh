// Token Importance Predictor scan (FASA: Frequency-aware Sparse Attention, §2.B.1).
//
// For KV head g of sequence b the score of cached token t is the fp32 dot of
//   q~_g = sum over the group's q heads of q_h, restricted to the dominant dims
//          {c, c + d/2 : c in I_dom[g]} (zero elsewhere)
// with the key row.  By linearity this is the per-head chunk sum of the method
// aggregated over the GQA group.  The kernel is a streaming GEMV: every key row
// is read once with 16-byte vector loads, S = row_bytes/16 lanes share a row and
// reduce with shuffles.  Two row sources:
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
  float* scores;            // [Hkv][T]
  int64_t row_stride_tok;   // elements between token rows of one head
  int64_t row_stride_head;  // elements between heads
  int32_t T, Hq, Hkv, d, G, n_dom;
  int32_t row_len;          // elements per row: k_dom cols (packed) or d (in place)
  int32_t packed;
  int32_t tile;             // tokens per CTA
  uint8_t heads[kMaxHeads]; // KV heads scored, one per blockIdx.y
};

__device__ __forceinline__ uint4 ld_stream_v4(const uint16_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float dot8(const uint4& w, const float (&qs)[8]) {
  float s = bf16lo(w.x) * qs[0];
  s = fmaf(bf16hi(w.x), qs[1], s);
  s = fmaf(bf16lo(w.y), qs[2], s);
  s = fmaf(bf16hi(w.y), qs[3], s);
  s = fmaf(bf16lo(w.z), qs[4], s);
  s = fmaf(bf16hi(w.z), qs[5], s);
  s = fmaf(bf16lo(w.w), qs[6], s);
  s = fmaf(bf16hi(w.w), qs[7], s);
  return s;
}

// S = lanes per row: row_len / 8 rounded up to a power of two (1 .. 16); lanes whose
// 16-byte segment lies past the row end carry zero weights and load nothing.
template <int S>
__global__ void __launch_bounds__(kTipThreads) tip_score_kernel(const TipParams p) {
  __shared__ float qt[128];
  const int b = blockIdx.z;
  const int g = p.heads[blockIdx.y];
  const int off = p.offsets[b];
  const int L = p.offsets[b + 1] - off;
  const int t0 = blockIdx.x * p.tile;
  if (t0 >= L) return;
  const int t1 = min(L, t0 + p.tile);
  const int C = p.d >> 1;
  const int tid = threadIdx.x;

  // q~ for this (b, g): fp32 group sum, restricted to the dominant dims.
  if (tid < p.row_len) {
    int dim = -1;
    if (p.packed) {
      if (tid < 2 * p.n_dom) {
        const int j = tid < p.n_dom ? tid : tid - p.n_dom;
        const int c = p.idom[g * p.n_dom + j];
        if (c < 0 || c >= C) {
          record_error(kCheckChunk, g, j, c);
        } else {
          dim = tid < p.n_dom ? c : c + C;
        }
      }
    } else if (p.idom == nullptr) {
      dim = tid;  // every chunk: the full dot
    } else {
      const int c = tid < C ? tid : tid - C;
      for (int j = 0; j < p.n_dom; ++j) {
        const int cj = p.idom[g * p.n_dom + j];
        if (cj < 0 || cj >= C) record_error(kCheckChunk, g, j, cj);
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

  const int lane = tid & 31;
  const int seg = lane % S;
  float qs[8];
  bool active = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    qs[i] = (seg * 8 + i < p.row_len) ? qt[seg * 8 + i] : 0.f;
    active |= (qs[i] != 0.f);
  }
  constexpr int RPI = kTipThreads / S;  // rows per block iteration
  constexpr int U = 8;                  // independent loads in flight per thread
  const uint16_t* base = p.src + (int64_t)g * p.row_stride_head + (int64_t)off * p.row_stride_tok + seg * 8;
  float* srow = p.scores + (int64_t)g * p.T + off;
  // Warp-uniform loop bounds: every lane of a warp takes the same trip count, so the
  // shuffles below always run with the full mask; rows past the tile are masked.
  const int warp_row0 = (tid >> 5) * (32 / S);
  const int lrow = lane / S;

  for (int tb = t0 + warp_row0; tb < t1; tb += U * RPI) {
    uint4 w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tt = tb + u * RPI + lrow;
      w[u] = make_uint4(0u, 0u, 0u, 0u);
      if (tt < t1 && active) w[u] = ld_stream_v4(base + (int64_t)tt * p.row_stride_tok);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float s = dot8(w[u], qs);
#pragma unroll
      for (int o = S / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const int tt = tb + u * RPI + lrow;
      if (seg == 0 && tt < t1) srow[tt] = s;
    }
  }
}

// ------------------------------------------------------------------ dominant-column packing
struct PackParams {
  const uint16_t* k;
  const int32_t* idom;
  uint16_t* k_dom;          // [Hkv][T][cols]
  int64_t stride_tok, stride_head;
  int32_t T, Hkv, d, n_dom, cols;
};

__global__ void __launch_bounds__(256) pack_dominant_kernel(const PackParams p) {
  const int C = p.d >> 1;
  const int64_t n_rows = (int64_t)p.Hkv * p.T;
  const int64_t total = n_rows * p.cols;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(e % p.cols);
    const int64_t row = e / p.cols;
    const int g = (int)(row / p.T);
    const int64_t t = row % p.T;
    uint16_t val = 0;
    if (j < 2 * p.n_dom) {
      const int c = p.idom[g * p.n_dom + (j < p.n_dom ? j : j - p.n_dom)];
      if (c < 0 || c >= C) {
        record_error(kCheckChunk, g, j, c);
      } else {
        const int dim = j < p.n_dom ? c : c + C;
        val = p.k[t * p.stride_tok + (int64_t)g * p.stride_head + dim];
      }
    }
    p.k_dom[e] = val;
  }
}

}  // namespace aoh
