// Appending a decoded token to the caches.
//
// AoH summary (Resumen Técnico: Autonomía de Cabezales), Metodología §4: retrieval
// heads keep the whole KV history, streaming heads keep only a fixed sink (the first
// tokens) and a recent window.  FASA: Frequency-aware Sparse Attention, §2.A: the key
// and query are rotated by RoPE at the token's absolute position (chunk c = dims
// (c, c + d/2), angle p * theta^(-2c/d)); §2.C: the dominant part of K is kept apart
// (here the packed dominant columns that the importance scan streams).
//
// One CTA per sequence b.  The new token's position is p = lengths[b] (the number of
// tokens the sequence held); after every row is written lengths[b] becomes p + 1.
//   * angles: p * theta^(-2c/d) and their sine / cosine in double precision, so the
//     rotation of a bf16 input is exact to far below one bf16 step at any position
//     (a single-precision angle would be off by ~1e-2 rad at p ~ 1e5);
//   * q and k are rotated with separately rounded double products (no fused
//     multiply-add), rounded to float and then to bf16 (nearest, ties to even);
//   * every KV head's K / V row goes to the cache(s) that store it: the linear cache
//     (token offsets[b] + p of its region) and / or the ring (slot ring_slot(p) of the
//     ring region; a ring without a window keeps no position past the sink);
//   * the packed dominant row of every head the linear cache stores, when it has one.
// A linear region already full, or a ring region smaller than its slots, writes
// nothing for that sequence and records device check 4.
#pragma once

#include "device_common.cuh"

namespace aoh {

constexpr int kAppendThreads = 256;

struct AppendParams {
  const uint16_t* q_new;      // [B][Hq][d] before rotation, or null
  const uint16_t* k_new;      // [B][Hkv][d] before rotation
  const uint16_t* v_new;      // [B][Hkv][d]
  uint16_t* q_out;            // [B][Hq][d] rotated, or null
  int32_t* lengths;           // [B]
  // linear cache (k null: none)
  uint16_t* k;
  uint16_t* v;
  const int32_t* offsets;
  int64_t stride_tok, stride_head;
  uint16_t* k_dom;            // [slots][T][k_dom_cols] or null
  int64_t T;
  int32_t k_dom_cols;
  const int32_t* idom;        // [Hkv][n_dom]
  int32_t n_dom;
  // ring cache (rk null: none)
  uint16_t* rk;
  uint16_t* rv;
  const int32_t* roffsets;
  int64_t rstride_tok, rstride_head;
  int32_t ring_sink, ring_window;
  int32_t B, Hq, Hkv, d;
  double theta;
  uint8_t slot[kMaxHeads];    // KV head -> slot in the linear cache (kNoSlot: not stored there)
  uint8_t rslot[kMaxHeads];   // KV head -> slot in the ring (kNoSlot: not stored there)
};

__device__ __forceinline__ double bf16_to_double(uint16_t h) { return (double)__uint_as_float((uint32_t)h << 16); }

__device__ __forceinline__ uint16_t double_to_bf16(double x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn((float)x));
}

// the rotated pair (u, v) of chunk c: (cos u - sin v, sin u + cos v), products rounded apart
__device__ __forceinline__ void rotate_pair(double u, double v, double cs, double sn, double* a, double* b) {
  *a = __dsub_rn(__dmul_rn(cs, u), __dmul_rn(sn, v));
  *b = __dadd_rn(__dmul_rn(sn, u), __dmul_rn(cs, v));
}

__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(const AppendParams p) {
  __shared__ double s_cos[64], s_sin[64];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int d = p.d, C = d >> 1;
  const int pos = p.lengths[b];
  // checks (uniform over the CTA: every thread reads the same values)
  if (pos < 0) {
    if (tid == 0) record_error(kCheckCapacity, b, pos, 0);
    return;
  }
  int64_t tok = -1, rtok = -1;
  if (p.k) {
    const int off = p.offsets[b], cap = p.offsets[b + 1] - off;
    if (pos >= cap) {
      if (tid == 0) record_error(kCheckCapacity, b, pos, cap);
      return;
    }
    tok = (int64_t)off + pos;
  }
  if (p.rk) {
    const int off = p.roffsets[b], cap = p.roffsets[b + 1] - off;
    if (cap < p.ring_sink + p.ring_window) {
      if (tid == 0) record_error(kCheckCapacity, b, cap, p.ring_sink + p.ring_window);
      return;
    }
    if (pos < p.ring_sink || p.ring_window > 0) rtok = (int64_t)off + ring_slot(pos, p.ring_sink, p.ring_window);
  }
  if (tid < C) {
    const double w = pow(p.theta, -2.0 * tid / d);
    sincos((double)pos * w, &s_sin[tid], &s_cos[tid]);
  }
  __syncthreads();

  // the query of every q head, rotated to the token's position
  if (p.q_new && p.q_out) {
    for (int e = tid; e < p.Hq * C; e += kAppendThreads) {
      const int h = e / C, c = e % C;
      const int64_t row = ((int64_t)b * p.Hq + h) * d;
      double a, bb;
      rotate_pair(bf16_to_double(p.q_new[row + c]), bf16_to_double(p.q_new[row + c + C]), s_cos[c], s_sin[c], &a, &bb);
      p.q_out[row + c] = double_to_bf16(a);
      p.q_out[row + c + C] = double_to_bf16(bb);
    }
  }
  // key rows (rotated) and value rows, into every cache that stores the head
  for (int e = tid; e < p.Hkv * C; e += kAppendThreads) {
    const int g = e / C, c = e % C;
    const int64_t row = ((int64_t)b * p.Hkv + g) * d;
    double a, bb;
    rotate_pair(bf16_to_double(p.k_new[row + c]), bf16_to_double(p.k_new[row + c + C]), s_cos[c], s_sin[c], &a, &bb);
    const uint16_t ka = double_to_bf16(a), kb = double_to_bf16(bb);
    const uint16_t va = p.v_new[row + c], vb = p.v_new[row + c + C];
    if (tok >= 0 && p.slot[g] != kNoSlot) {
      const int64_t o = tok * p.stride_tok + (int64_t)p.slot[g] * p.stride_head;
      p.k[o + c] = ka;
      p.k[o + c + C] = kb;
      p.v[o + c] = va;
      p.v[o + c + C] = vb;
    }
    if (rtok >= 0 && p.rslot[g] != kNoSlot) {
      const int64_t o = rtok * p.rstride_tok + (int64_t)p.rslot[g] * p.rstride_head;
      p.rk[o + c] = ka;
      p.rk[o + c + C] = kb;
      p.rv[o + c] = va;
      p.rv[o + c + C] = vb;
    }
  }
  // the packed dominant row (columns: dims I_dom, then I_dom + d/2, then zeros)
  if (tok >= 0 && p.k_dom) {
    for (int e = tid; e < p.Hkv * p.k_dom_cols; e += kAppendThreads) {
      const int g = e / p.k_dom_cols, j = e % p.k_dom_cols;
      if (p.slot[g] == kNoSlot) continue;
      uint16_t val = 0;
      if (j < 2 * p.n_dom) {
        const int c = p.idom[g * p.n_dom + (j < p.n_dom ? j : j - p.n_dom)];
        if (c < 0 || c >= C) {
          record_error(kCheckChunk, g, j, c);
        } else {
          const int64_t row = ((int64_t)b * p.Hkv + g) * d;
          double a, bb;
          rotate_pair(bf16_to_double(p.k_new[row + c]), bf16_to_double(p.k_new[row + c + C]), s_cos[c], s_sin[c], &a,
                      &bb);
          val = double_to_bf16(j < p.n_dom ? a : bb);
        }
      }
      p.k_dom[((int64_t)p.slot[g] * p.T + tok) * p.k_dom_cols + j] = val;
    }
  }
  __syncthreads();
  if (tid == 0) p.lengths[b] = pos + 1;
}

}  // namespace aoh
