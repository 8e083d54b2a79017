// Top-N_fac selection over precomputed scores, spread over chunks of every row
// (FASA: Frequency-aware Sparse Attention, §2.B.1, keep the N_fac best tokens; the
// shared index of "Cómo funciona CLSA" is the same operation with k fixed).
//
// Keys are the order-preserving uint32 images of the fp32 scores (-0 folded onto +0).
// The selection of a (sequence b, KV head g) row is {key > K_T} plus the lowest
// positions among {key == K_T}, n in all, written in ascending position order.
//
// First digit: the top 11 bits of a key (sign, exponent, two mantissa bits).  The row's
// histogram of it comes from the importance scan (which counts each score as it writes
// it) or, on caller-given scores, from select_hist_kernel.  Then, with chunks of
// kSelChunk keys of a row, one CTA each:
//   select_chunk_kernel  finds the bin T1 holding the n-th key from the histogram, counts
//                        the chunk's keys above T1 and appends the chunk's keys in T1
//                        (key, position) to the row's candidate list.  The last CTA of the
//                        row (atomic ticket) resolves K_T among the candidates with the
//                        remaining 21 bits (digits of 8, 8 and 5 bits), counts per chunk the
//                        candidates above and equal to K_T, and turns all counts into every
//                        chunk's output offset and number of equal keys before it; it then
//                        re-arms the histogram, the candidate count and the ticket to zero;
//   select_write_kernel  every chunk writes its selected positions at its offset, in order:
//                        warps own runs of 32 x kWriteK consecutive keys, ballots rank the
//                        picks inside a warp, one block scan ranks the warps.
// A row with n >= L_b takes every position without a select.  Deterministic: the
// candidate list's order varies between runs, the counts drawn from it do not.
#pragma once

#include "device_common.cuh"

namespace aoh {

constexpr int kSelChunk = 4096;        // keys of a row per CTA
constexpr int kSelHistBins = 2048;     // first digit: the top 11 bits of a key
constexpr int kSelHistShift = 21;
constexpr int kSelCtaThreads = 256;
constexpr int kWriteK = kSelChunk / kSelCtaThreads;  // keys per lane in the write pass (16)
constexpr int kSelMaxChunks = 1024;    // chunks per row: rows up to 4 M keys
constexpr int kSelResolveCap = 8192;   // candidates the last CTA keeps in shared memory

struct HistSelectParams {
  const float* scores;          // [Hkv][T]
  const int32_t* offsets;       // [B + 1]
  const int32_t* lengths;       // [B] or null
  const int32_t* n_fac_per_seq; // [B] or null
  uint32_t* hist;               // [Hkv][B][2048], zero between calls
  unsigned long long* cand;     // [Hkv][T]: (key << 32 | position) of the row at offset offsets[b]
  int32_t* cand_count;          // [Hkv][B], zero between calls
  int32_t* tickets;             // [Hkv][B], zero between calls
  int32_t* chunk_above;         // [Hkv][B][max_chunks]
  int32_t* chunk_info;          // [Hkv][B][max_chunks][2]: selected before the chunk, equal keys before it
  int32_t* row_info;            // [Hkv][B][2]: K_T, equal keys taken
  int32_t* idx;                 // [B][Hkv][cap]
  int32_t* count;               // [B][Hkv]
  int32_t T, B, Hkv, n_fac, cap, max_chunks;
  uint8_t heads[kMaxHeads];     // KV head of blockIdx.y
};

__device__ __forceinline__ int sel_n(const HistSelectParams& p, int b, int L, bool report) {
  int nf = p.n_fac_per_seq ? p.n_fac_per_seq[b] : p.n_fac;
  if (nf > p.cap) {
    if (report) record_error(kCheckCount, b, nf, p.cap);
    nf = p.cap;
  }
  return max(0, min(nf, L));
}

// ---------------------------------------------------------------------------- histogram
// The first-digit histogram of the chunk's keys, added into the row's global histogram
// (non-empty bins only).
__global__ void __launch_bounds__(kSelCtaThreads) select_hist_kernel(const HistSelectParams p) {
  __shared__ uint32_t h[kSelHistBins];
  const int c = blockIdx.x, g = p.heads[blockIdx.y], b = blockIdx.z, tid = threadIdx.x;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  const int n = sel_n(p, b, L, false);
  if (n >= L || c * kSelChunk >= L) return;  // nothing to select here
  for (int i = tid; i < kSelHistBins; i += kSelCtaThreads) h[i] = 0u;
  __syncthreads();
  const float* row = p.scores + (int64_t)g * p.T + off;
  const int i1 = min(L, (c + 1) * kSelChunk);
  for (int i = c * kSelChunk + tid; i < i1; i += kSelCtaThreads) atomicAdd(&h[score_key(__ldcg(row + i)) >> kSelHistShift], 1u);
  __syncthreads();
  uint32_t* gh = p.hist + ((int64_t)g * p.B + b) * kSelHistBins;
  for (int i = tid; i < kSelHistBins; i += kSelCtaThreads)
    if (h[i]) atomicAdd(gh + i, h[i]);
}

// The bin holding the n-th largest key of a row, from its histogram: every thread takes 8
// bins from the top down.  Returns T1; *above = keys in higher bins.  Called by every thread.
__device__ __forceinline__ int threshold_bin(const uint32_t* gh, int n, int* above, int* scratch, int* s_out) {
  const int tid = threadIdx.x;
  constexpr int per = kSelHistBins / kSelCtaThreads;  // 8
  if (tid == 0) {  // kept only if the histogram holds fewer than n keys (it holds the row's L >= n)
    s_out[0] = 0;
    s_out[1] = 0;
  }
  int cnt[per], tot = 0;
#pragma unroll
  for (int k = 0; k < per; ++k) {
    cnt[k] = (int)__ldcg(gh + (kSelHistBins - 1 - (tid * per + k)));  // bin order: top first
    tot += cnt[k];
  }
  int total;
  int excl = block_exclusive_scan(tot, scratch, &total);
  if (tid == 0 && total < n) record_error(kCheckCount, n, total, -2);
  if (excl < n && n <= excl + tot) {
#pragma unroll
    for (int k = 0; k < per; ++k) {
      if (excl < n && n <= excl + cnt[k]) {
        s_out[0] = kSelHistBins - 1 - (tid * per + k);
        s_out[1] = excl;
      }
      excl += cnt[k];
    }
  }
  __syncthreads();
  *above = s_out[1];
  return s_out[0];
}

// ---------------------------------------------------------------------------- chunk pass
__global__ void __launch_bounds__(kSelCtaThreads) select_chunk_kernel(const HistSelectParams p) {
  __shared__ int scratch[33];
  __shared__ int s_out[2];
  __shared__ int s_last;
  __shared__ int s_warp[kSelCtaThreads / 32];
  __shared__ uint32_t s_key[kSelResolveCap];
  __shared__ int s_hist[256];
  __shared__ int s_gt[kSelMaxChunks], s_eq[kSelMaxChunks];  // per-chunk counts
  const int c = blockIdx.x, g = p.heads[blockIdx.y], b = blockIdx.z, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  const int n = sel_n(p, b, L, c == 0 && tid == 0);
  const int nch = (L + kSelChunk - 1) / kSelChunk;
  const int64_t rid = (int64_t)g * p.B + b;
  uint32_t* gh = p.hist + rid * kSelHistBins;
  if (n >= L) {  // every position taken: the write pass alone; the scan's counts are cleared
    if (c == 0)
      for (int i = tid; i < kSelHistBins; i += kSelCtaThreads) gh[i] = 0u;
    return;
  }
  if (c >= nch) return;
  int above1;
  const int T1 = threshold_bin(gh, n, &above1, scratch, s_out);

  // this chunk: keys above the bin (counted), keys in the bin (to the candidate list)
  const float* row = p.scores + (int64_t)g * p.T + off;
  unsigned long long* cand = p.cand + (int64_t)g * p.T + off;
  const int i0 = c * kSelChunk, i1 = min(L, i0 + kSelChunk);
  int n_above = 0;
  uint32_t kk[kWriteK];
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {  // every load in flight before any is used
    const int i = i0 + r * kSelCtaThreads + tid;
    kk[r] = i < i1 ? score_key(__ldcg(row + i)) : 0u;
  }
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    const int i = i0 + r * kSelCtaThreads + tid;
    const uint32_t k = kk[r];
    const int bin = (int)(k >> kSelHistShift);
    n_above += (i < i1 && bin > T1);
    const bool hit = i < i1 && bin == T1;
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    int wbase = 0;
    if (lane == 0 && bal) wbase = atomicAdd(p.cand_count + rid, __popc(bal));
    wbase = __shfl_sync(0xffffffffu, wbase, 0);
    if (hit) cand[wbase + __popc(bal & ((1u << lane) - 1u))] = ((unsigned long long)k << 32) | (uint32_t)i;
  }
  n_above = __reduce_add_sync(0xffffffffu, n_above);
  if (lane == 0) s_warp[warp] = n_above;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < kSelCtaThreads / 32; ++w) t += s_warp[w];
    p.chunk_above[rid * p.max_chunks + c] = t;
  }
  // ---- the last CTA of the row resolves K_T
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(p.tickets + rid, 1) == nch - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int m = atomicAdd(p.cand_count + rid, 0);  // every candidate of the row is written
  const bool in_smem = m <= kSelResolveCap;
  if (in_smem) {
    for (int j = tid; j < m; j += kSelCtaThreads) s_key[j] = (uint32_t)(__ldcg(cand + j) >> 32);
    __syncthreads();
  }
  // rank krem (1 = largest) among the candidates, digits of the low 21 bits
  uint32_t prefix = (uint32_t)T1 << kSelHistShift, pmask = 0xffffffffu << kSelHistShift;
  int krem = n - above1;
  const int shifts[3] = {13, 5, 0};
  const int widths[3] = {8, 8, 5};
#pragma unroll 1
  for (int d = 0; d < 3; ++d) {
    const int sh = shifts[d], nb = 1 << widths[d];
    if (tid < 256) s_hist[tid] = 0;
    __syncthreads();
    for (int j = tid; j < m; j += kSelCtaThreads) {
      const uint32_t k = in_smem ? s_key[j] : (uint32_t)(__ldcg(cand + j) >> 32);
      if ((k & pmask) == prefix) atomicAdd(&s_hist[(k >> sh) & (nb - 1)], 1);
    }
    __syncthreads();
    // bins from the top: thread t takes bin nb - 1 - t
    const int cnt = tid < nb ? s_hist[nb - 1 - tid] : 0;
    int total;
    const int excl = block_exclusive_scan(cnt, scratch, &total);
    if (tid < nb && excl < krem && krem <= excl + cnt) {
      s_out[0] = nb - 1 - tid;
      s_out[1] = excl;
    }
    __syncthreads();
    prefix |= (uint32_t)s_out[0] << sh;
    pmask |= (uint32_t)(nb - 1) << sh;
    krem -= s_out[1];
    __syncthreads();
  }
  const uint32_t KT = prefix;
  const int need_eq = krem;  // keys equal to K_T that are taken (>= 1), lowest positions first
  // candidates above / equal to K_T, per chunk
  for (int q = tid; q < nch; q += kSelCtaThreads) {
    s_gt[q] = 0;
    s_eq[q] = 0;
  }
  __syncthreads();
  for (int j = tid; j < m; j += kSelCtaThreads) {
    const unsigned long long e = __ldcg(cand + j);
    const uint32_t k = (uint32_t)(e >> 32);
    const int q = (int)(uint32_t)e / kSelChunk;
    if (k > KT) atomicAdd(&s_gt[q], 1);
    else if (k == KT) atomicAdd(&s_eq[q], 1);
  }
  __syncthreads();
  // offsets: thread t owns chunks [t * per, (t + 1) * per)
  const int per = (nch + kSelCtaThreads - 1) / kSelCtaThreads;
  int sel_t = 0, eq_t = 0;
  for (int q = tid * per; q < min(nch, (tid + 1) * per); ++q) {
    sel_t += __ldcg(p.chunk_above + rid * p.max_chunks + q) + s_gt[q];
    eq_t += s_eq[q];
  }
  int tot_sel, tot_eq;
  int sel_before = block_exclusive_scan(sel_t, scratch, &tot_sel);
  int eq_before = block_exclusive_scan(eq_t, scratch, &tot_eq);
  for (int q = tid * per; q < min(nch, (tid + 1) * per); ++q) {
    // selected before chunk q: keys above K_T before it plus the equal keys taken before it
    p.chunk_info[(rid * p.max_chunks + q) * 2] = sel_before + min(need_eq, eq_before);
    p.chunk_info[(rid * p.max_chunks + q) * 2 + 1] = eq_before;
    sel_before += __ldcg(p.chunk_above + rid * p.max_chunks + q) + s_gt[q];
    eq_before += s_eq[q];
  }
  if (tid == 0) {
    p.row_info[rid * 2] = (int)KT;
    p.row_info[rid * 2 + 1] = need_eq;
    p.cand_count[rid] = 0;
    p.tickets[rid] = 0;
  }
  for (int i = tid; i < kSelHistBins; i += kSelCtaThreads) gh[i] = 0u;
}

// ---------------------------------------------------------------------------- ordered write
__global__ void __launch_bounds__(kSelCtaThreads) select_write_kernel(const HistSelectParams p) {
  __shared__ int scratch[33];
  const int c = blockIdx.x, g = p.heads[blockIdx.y], b = blockIdx.z, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  const int n = sel_n(p, b, L, false);
  int32_t* out = p.idx + ((int64_t)b * p.Hkv + g) * p.cap;
  if (c == 0) {
    for (int j = n + tid; j < p.cap; j += kSelCtaThreads) out[j] = -1;
    if (tid == 0) p.count[(int64_t)b * p.Hkv + g] = n;
  }
  const int i0 = c * kSelChunk;
  if (i0 >= L || n == 0) return;
  const int i1 = min(L, i0 + kSelChunk);
  if (n >= L) {  // every position, in order
    for (int i = i0 + tid; i < i1; i += kSelCtaThreads) out[i] = i;
    return;
  }
  const int64_t rid = (int64_t)g * p.B + b;
  const uint32_t KT = (uint32_t)__ldcg(p.row_info + rid * 2);
  const int need_eq = __ldcg(p.row_info + rid * 2 + 1);
  const int sel_chunk = __ldcg(p.chunk_info + (rid * p.max_chunks + c) * 2);
  const int eq_chunk = __ldcg(p.chunk_info + (rid * p.max_chunks + c) * 2 + 1);
  const float* row = p.scores + (int64_t)g * p.T + off;
  // warp w owns keys [i0 + w * 32 * kWriteK, ...): lane-consecutive loads, kWriteK rounds
  const int w0 = i0 + warp * 32 * kWriteK;
  uint32_t k[kWriteK];
  int ngt = 0, neq = 0;
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    const int i = w0 + r * 32 + lane;
    k[r] = i < i1 ? score_key(__ldcg(row + i)) : 0u;
    ngt += (i < i1 && k[r] > KT);
    neq += (i < i1 && k[r] == KT);
  }
  ngt = __reduce_add_sync(0xffffffffu, ngt);
  neq = __reduce_add_sync(0xffffffffu, neq);
  int tot;
  // warp offsets inside the chunk (lane 0 of each warp contributes its warp's counts)
  const int packed = block_exclusive_scan(lane == 0 ? ((ngt << 16) | neq) : 0, scratch, &tot);
  int gt_before = __shfl_sync(0xffffffffu, packed >> 16, 0);
  int eq_before = eq_chunk + __shfl_sync(0xffffffffu, packed & 0xffff, 0);
  // equal keys taken before this warp, and selected keys before it
  int sel_before = sel_chunk + gt_before + (min(need_eq, eq_before) - min(need_eq, eq_chunk));
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    const int i = w0 + r * 32 + lane;
    const bool in = i < i1;
    const bool gt = in && k[r] > KT;
    const bool eq = in && k[r] == KT;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_before + __popc(beq & ((1u << lane) - 1u));
    const bool take = gt || (eq && eq_rank < need_eq);
    const unsigned bt = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int o = sel_before + __popc(bt & ((1u << lane) - 1u));
      if (o < n) out[o] = i;  // o < n by construction; kept as a guard
    }
    sel_before += __popc(bt);
    eq_before += __popc(beq);
  }
}

}  // namespace aoh
