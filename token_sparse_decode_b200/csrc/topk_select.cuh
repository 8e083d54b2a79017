// Top-N_fac selection over precomputed scores (FASA: Frequency-aware Sparse
// Attention, §2.B.1; the shared index of "Cómo funciona CLSA" is the same
// operation with k fixed).
//
// One CTA of 512 threads per (sequence b, KV head g) row; the row's fp32 scores
// (written by the scan kernel just before, so resident in L2) are read as
// order-preserving uint32 keys.  An MSB-first radix select (4 digits of 8 bits)
// finds the n-th largest key K_T:
//   digit 0: a coalesced pass over the row builds per-warp 256-bin histograms
//            (plain shared-memory atomics), which also give every warp its offset
//            for the compaction below;
//   then the keys sharing the chosen first digit are compacted into shared
//            memory by a second pass (when they fit; otherwise the later digits
//            re-read the row), and digits 1-3 are counted over those candidates.
// The selection is {key > K_T} plus the first (n - #{key > K_T}) positions with
// key == K_T in position order, i.e. "score descending, lower position first".
// A third pass writes it in ascending position order: tiles of 2048 positions,
// four consecutive positions per thread, one block scan of the packed
// (#greater, #equal) counts per tile gives each thread its output offset and
// its rank among the equal keys.  Deterministic; no cluster, no global scratch.
#pragma once

#include "device_common.cuh"

namespace aoh {

constexpr int kSelThreads = 512;
constexpr int kSelCandCap = 20480;  // candidate keys kept in shared memory (80 KB: two CTAs an SM)
constexpr int kSelU = 8;            // row loads in flight per lane in the streaming passes

struct SelectParams {
  const float* scores;            // [Hkv][T]
  const int32_t* offsets;         // [B + 1]
  const int32_t* lengths;         // [B] or null (sequences fill their regions)
  const int32_t* n_fac_per_seq;   // [B] or null
  int32_t* idx;                   // [B][Hkv][cap]
  int32_t* count;                 // [B][Hkv]
  int32_t T, Hkv, n_fac, cap;
  uint8_t heads[kMaxHeads];       // KV head of blockIdx.x
  uint8_t slot[kMaxHeads];        // head slots of the cache (the scores are indexed by KV head)
};

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(const SelectParams p) {
  extern __shared__ __align__(16) uint32_t cand[];  // kSelCandCap keys
  __shared__ int hist[256];
  __shared__ int whist[kSelThreads / 32][256];  // per-warp first-digit counts (and candidate offsets)
  __shared__ int scan_scratch[33];
  __shared__ int s_bin, s_above, s_in_bin;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y;
  const int g = p.heads[blockIdx.x];
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  int nf = p.n_fac_per_seq ? p.n_fac_per_seq[b] : p.n_fac;
  if (nf > p.cap) {
    if (tid == 0) record_error(kCheckCount, b, nf, p.cap);
    nf = p.cap;
  }
  const int n = max(0, min(nf, L));
  int32_t* out = p.idx + ((int64_t)b * p.Hkv + g) * p.cap;
  const float* row = p.scores + (int64_t)g * p.T + off;
  for (int j = n + tid; j < p.cap; j += kSelThreads) out[j] = -1;
  if (tid == 0) p.count[(int64_t)b * p.Hkv + g] = n;
  if (n == 0) return;  // before any barrier: uniform over the CTA
  // N_fac >= L needs no special case: the threshold is then the smallest key and every
  // key equal to it is taken, so the compaction below writes every position in order.

  // ---- threshold K_T: 4 digits of 8 bits, most significant first
  uint32_t prefix = 0u, pmask = 0u;
  int krem = n;        // rank of the threshold among the keys matching the prefix (1 = largest)
  int nc = -1;         // candidates in shared memory (-1: the row is re-read)
  int eq_total = 0;    // keys equal to K_T (the chosen bin of the last digit)
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0;
    if (pass == 0)
      for (int i = tid; i < (kSelThreads / 32) * 256; i += kSelThreads) (&whist[0][0])[i] = 0;
    __syncthreads();
    if (nc >= 0) {
      for (int i = tid; i < nc; i += kSelThreads) {
        const uint32_t k = cand[i];
        if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
      }
    } else {
      // coalesced pass over the row, eight loads in flight per lane; plain shared-memory
      // atomics (the first digit into this warp's histogram)
      int* h = pass == 0 ? whist[warp] : hist;
      for (int base = warp * 32; base < L; base += kSelU * kSelThreads) {
        float v[kSelU];
#pragma unroll
        for (int u = 0; u < kSelU; ++u) {
          const int i = base + u * kSelThreads + lane;
          v[u] = i < L ? __ldcg(row + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kSelU; ++u) {
          const int i = base + u * kSelThreads + lane;
          const uint32_t k = score_key(v[u]);
          if (i < L && (k & pmask) == prefix) atomicAdd(&h[(k >> shift) & 255u], 1);
        }
      }
      if (pass == 0) {
        __syncthreads();
        if (tid < 256) {
          int c = 0;
#pragma unroll
          for (int w2 = 0; w2 < kSelThreads / 32; ++w2) c += whist[w2][tid];
          hist[tid] = c;
        }
      }
    }
    __syncthreads();
    // bins from the top down: exclusive prefix, then the bin holding rank krem
    const int tot = tid < 256 ? hist[255 - tid] : 0;
    int total;
    const int above = block_exclusive_scan(tot, scan_scratch, &total);
    if (tid < 256 && above < krem && krem <= above + tot) {
      s_bin = 255 - tid;
      s_above = above;
      s_in_bin = tot;
    }
    __syncthreads();
    prefix |= (uint32_t)s_bin << shift;
    pmask |= 255u << shift;
    krem -= s_above;
    eq_total = s_in_bin;
    // after the first digit: compact the keys sharing it (order irrelevant: only counted).
    // Every warp writes from its own offset: the counts of the chosen bin in the lower warps.
    const bool compact = (pass == 0) && (s_in_bin <= kSelCandCap);
    if (compact) {
      int wbase = 0;
      for (int w2 = 0; w2 < warp; ++w2) wbase += whist[w2][s_bin];
      for (int base = warp * 32; base < L; base += kSelU * kSelThreads) {
        float v[kSelU];
#pragma unroll
        for (int u = 0; u < kSelU; ++u) {
          const int i = base + u * kSelThreads + lane;
          v[u] = i < L ? __ldcg(row + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kSelU; ++u) {
          const int i = base + u * kSelThreads + lane;
          const uint32_t k = score_key(v[u]);
          const bool hit = i < L && (k & pmask) == prefix;
          const unsigned bal = __ballot_sync(0xffffffffu, hit);
          if (hit) cand[wbase + __popc(bal & ((1u << lane) - 1u))] = k;
          wbase += __popc(bal);
        }
      }
    }
    const int n_in = s_in_bin;
    __syncthreads();
    if (compact) nc = n_in;
  }
  const uint32_t KT = prefix;
  const int need_eq = krem;    // keys equal to K_T that are taken, lowest positions first

  // ---- ordered compaction: tiles of 4 * kSelThreads positions, 4 consecutive per thread
  int sel_base = 0, eq_base = 0;
  const bool all_eq = (eq_total == need_eq);  // every key equal to K_T is taken
  // the next tile's scores are loaded while this tile is scanned
  float vn[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) vn[j] = 4 * tid + j < L ? __ldg(row + 4 * tid + j) : 0.f;
  for (int t0 = 0; t0 < L; t0 += 4 * kSelThreads) {
    const int i0 = t0 + 4 * tid;
    uint32_t k[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) k[j] = score_key(vn[j]);
    const int i1 = i0 + 4 * kSelThreads;
#pragma unroll
    for (int j = 0; j < 4; ++j) vn[j] = i1 + j < L ? __ldg(row + i1 + j) : 0.f;  // L1 merges the 4 strided loads
    int ngt = 0, neq = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool in = i0 + j < L;
      ngt += (in && k[j] > KT);
      neq += (in && k[j] == KT);
    }
    int packed_tot;
    const int packed = block_exclusive_scan((ngt << 16) | neq, scan_scratch, &packed_tot);
    const int gt_excl = packed >> 16, eq_excl = packed & 0xffff;
    // equal keys before this thread (whole row), and how many of them are taken
    const int eq_prev = eq_base + eq_excl;
    int pos = sel_base + gt_excl + (all_eq ? eq_excl : min(need_eq, eq_prev) - min(need_eq, eq_base));
    int eq_seen = eq_prev;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (i0 + j >= L) break;
      bool take = k[j] > KT;
      if (k[j] == KT) {
        take = all_eq || eq_seen < need_eq;
        ++eq_seen;
      }
      if (take) {
        if (pos < n) out[pos] = i0 + j;  // pos < n by construction; kept as a guard
        ++pos;
      }
    }
    const int gt_t = packed_tot >> 16, eq_t = packed_tot & 0xffff;
    sel_base += gt_t + (all_eq ? eq_t : min(need_eq, eq_base + eq_t) - min(need_eq, eq_base));
    eq_base += eq_t;
  }
}

}  // namespace aoh
