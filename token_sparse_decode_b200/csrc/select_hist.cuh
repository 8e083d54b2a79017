// Top-N_fac selection over precomputed scores, spread over chunks of every row
// (FASA: Frequency-aware Sparse Attention, §2.B.1, keep the N_fac best tokens; the
// shared index of "Cómo funciona CLSA" is the same operation with k fixed).
//
// Keys are the order-preserving uint32 images of the fp32 scores (-0 folded onto +0).
// The selection of a (sequence b, KV head g) row is {key > K_T} plus the lowest
// positions among {key == K_T}, n in all, written in ascending position order.
//
// First digit: the top 11 bits of a key (sign, exponent, two mantissa bits).  Four phases
// over chunks of kSelChunk keys of every row (the resolve over rows):
//   hist     counts a chunk's first digits in shared memory and adds the non-empty bins
//            into the row's histogram (chunk 0 also clears the row's candidate count);
//   chunk    finds the bin T1 holding the n-th key from the histogram (chunk 0 records T1
//            and the keys above it for the row), counts the chunk's keys above T1 and
//            appends its keys in T1 (key, position) to the row's candidate list (one
//            atomic per CTA reserves the chunk's run of the list);
//   resolve  per row: the exact threshold among the candidates (the remaining 21 bits in
//            digits of 11 and 10; when the chosen bin holds exactly the keys still needed
//            its low bits do not matter, the bin is taken whole and keys are compared
//            masked), every chunk's output offset and number of equal keys before it;
//            re-arms the row's histogram to zero;
//   write    a chunk's selected positions at its offset, in order: warps own runs of
//            32 x kWriteK consecutive keys, ballots rank the picks inside a warp, one
//            block scan ranks the warps.
// One kernel per phase (four launches, each dependency a kernel boundary); the phase bodies
// are item functions over one shared scratch buffer.  Every phase issues all of its key
// loads before it uses any.  A row with n >= L_b takes every position
// without a select.  Deterministic: the candidate list's order varies between runs, the
// counts drawn from it do not.
#pragma once

#include "device_common.cuh"

namespace aoh {

constexpr int kSelChunk = 4096;        // keys of a row per chunk
constexpr int kSelHistBins = 2048;     // first digit: the top 11 bits of a key
constexpr int kSelHistShift = 21;
constexpr int kSelCtaThreads = 256;
constexpr int kWriteK = kSelChunk / kSelCtaThreads;  // keys per lane (16)
constexpr int kSelMaxChunks = 1024;    // chunks per row: rows up to 4 M keys
constexpr int kSelResolveCap = 4096;   // candidates the resolve keeps in shared memory (more: read from L2)
constexpr int kRowInfo = 8;            // ints per row in row_info
// shared scratch of the resolve phase
constexpr int kSelSmem = 144 + 4 * kSelHistBins + 4 * kSelResolveCap + 2 * kSelResolveCap + 8 * kSelMaxChunks;

struct HistSelectParams {
  const float* scores;          // [Hkv][T]
  const int32_t* offsets;       // [B + 1]
  const int32_t* lengths;       // [B] or null
  const int32_t* n_fac_per_seq; // [B] or null
  uint32_t* hist;               // [Hkv][B][2048], zero between calls
  unsigned long long* cand;     // [Hkv][T]: (key << 32 | position) of the row at offset offsets[b]
  int32_t* cand_count;          // [Hkv][B]
  int32_t* chunk_above;         // [Hkv][B][max_chunks]: keys of the chunk above T1
  int32_t* chunk_info;          // [Hkv][B][max_chunks][2]: keys selected before the chunk, equal keys before it
  int32_t* row_info;            // [Hkv][B][kRowInfo]: T1, keys above T1, threshold prefix, its mask, equal keys taken
  int32_t* idx;                 // [B][Hkv][cap]
  int32_t* count;               // [B][Hkv]
  int32_t T, B, Hkv, n_fac, cap, max_chunks;
  uint8_t heads[kMaxHeads];     // listed KV heads
};

__device__ __forceinline__ int sel_n(const HistSelectParams& p, int b, int L, bool report) {
  int nf = p.n_fac_per_seq ? p.n_fac_per_seq[b] : p.n_fac;
  if (nf > p.cap) {
    if (report) record_error(kCheckCount, b, nf, p.cap);
    nf = p.cap;
  }
  return max(0, min(nf, L));
}

// ---------------------------------------------------------------------------- hist phase
// The first-digit histogram of chunk c of row (listed head y, sequence b), added into the
// row's global histogram (non-empty bins only).
__device__ __forceinline__ void sel_hist_item(const HistSelectParams& p, uint8_t* sm, int c, int y, int b) {
  uint32_t* h = reinterpret_cast<uint32_t*>(sm);
  const int g = p.heads[y], tid = threadIdx.x;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  const int n = sel_n(p, b, L, false);
  if (n == 0 || n >= L || c * kSelChunk >= L) return;  // nothing to select here
  const float* row = p.scores + (int64_t)g * p.T + off;
  const int i0 = c * kSelChunk, i1 = min(L, i0 + kSelChunk);
  float f[kWriteK];
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {  // every load in flight before any is used
    const int i = i0 + r * kSelCtaThreads + tid;
    f[r] = i < i1 ? __ldcg(row + i) : 0.f;
  }
  if (c == 0 && tid == 0) p.cand_count[(int64_t)g * p.B + b] = 0;  // read after this phase only
  __syncthreads();  // the scratch may still be read for the previous item
  for (int i = tid; i < kSelHistBins; i += kSelCtaThreads) h[i] = 0u;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kWriteK; ++r)
    if (i0 + r * kSelCtaThreads + tid < i1) atomicAdd(&h[score_key(f[r]) >> kSelHistShift], 1u);
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

// ---------------------------------------------------------------------------- chunk phase
__device__ __forceinline__ void sel_chunk_item(const HistSelectParams& p, uint8_t* sm, int c, int y, int b) {
  int* scratch = reinterpret_cast<int*>(sm);  // [33]
  int* s_out = scratch + 33;                  // [2]
  int* s_warp = s_out + 2;                    // [8]
  int* s_whit = s_warp + 8;                   // [8]
  int* s_base = s_whit + 8;                   // [1]
  const int g = p.heads[y], tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  const int n = sel_n(p, b, L, c == 0 && tid == 0);
  const int nch = (L + kSelChunk - 1) / kSelChunk;
  const int64_t rid = (int64_t)g * p.B + b;
  if (n == 0 || n >= L || c >= nch) return;  // nothing to select (the write phase alone), or past the row
  // this chunk's keys first: their loads fly while the row's histogram is read
  const float* row = p.scores + (int64_t)g * p.T + off;
  unsigned long long* cand = p.cand + (int64_t)g * p.T + off;
  const int i0 = c * kSelChunk, i1 = min(L, i0 + kSelChunk);
  uint32_t kk[kWriteK];
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    const int i = i0 + r * kSelCtaThreads + tid;
    kk[r] = i < i1 ? score_key(__ldcg(row + i)) : 0u;
  }
  __syncthreads();  // the scratch may still be read for the previous item
  int above1;
  const int T1 = threshold_bin(p.hist + rid * kSelHistBins, n, &above1, scratch, s_out);
  if (c == 0 && tid == 0) {
    p.row_info[rid * kRowInfo] = T1;
    p.row_info[rid * kRowInfo + 1] = above1;
  }
  // keys above the bin (counted) and keys in the bin (to the candidate list: one atomic per
  // CTA reserves the chunk's run, warps and lanes take consecutive places in it)
  int n_above = 0, n_hit = 0;
  unsigned hits[kWriteK];
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    const int i = i0 + r * kSelCtaThreads + tid;
    const int bin = (int)(kk[r] >> kSelHistShift);
    n_above += (i < i1 && bin > T1);
    hits[r] = __ballot_sync(0xffffffffu, i < i1 && bin == T1);
    n_hit += __popc(hits[r]);
  }
  n_above = __reduce_add_sync(0xffffffffu, n_above);
  if (lane == 0) {
    s_warp[warp] = n_above;
    s_whit[warp] = n_hit;
  }
  __syncthreads();
  if (tid == 0) {
    int t = 0, hsum = 0;
    for (int w = 0; w < kSelCtaThreads / 32; ++w) {
      t += s_warp[w];
      const int x = s_whit[w];
      s_whit[w] = hsum;  // exclusive offsets of the warps' candidates
      hsum += x;
    }
    p.chunk_above[rid * p.max_chunks + c] = t;
    s_base[0] = hsum ? atomicAdd(p.cand_count + rid, hsum) : 0;
  }
  __syncthreads();
  int wbase = s_base[0] + s_whit[warp];
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    if ((hits[r] >> lane) & 1u)
      cand[wbase + __popc(hits[r] & ((1u << lane) - 1u))] =
          ((unsigned long long)kk[r] << 32) | (uint32_t)(i0 + r * kSelCtaThreads + tid);
    wbase += __popc(hits[r]);
  }
}

// ---------------------------------------------------------------------------- resolve phase
// Row (listed head y, sequence b): the exact threshold among the row's candidates, then every
// chunk's output offset: the keys above T1 in the chunks before it, their candidates above
// the threshold and the equal keys taken before it.  Re-arms the row's histogram (its last
// reader was the chunk phase).
__device__ __forceinline__ void sel_resolve_row(const HistSelectParams& p, uint8_t* sm, int y, int b) {
  int* scratch = reinterpret_cast<int*>(sm);                             // [33]
  int* s_out = scratch + 33;                                             // [3]
  int* s_hist = reinterpret_cast<int*>(sm + 144);                        // [2048]
  uint32_t* s_key = reinterpret_cast<uint32_t*>(sm + 144 + 4 * kSelHistBins);  // [kSelResolveCap]
  uint16_t* s_chk = reinterpret_cast<uint16_t*>(s_key + kSelResolveCap);        // [kSelResolveCap]
  int* s_gt = reinterpret_cast<int*>(s_chk + kSelResolveCap);                   // [kSelMaxChunks]
  int* s_eq = s_gt + kSelMaxChunks;                                             // [kSelMaxChunks]
  constexpr int NT = kSelCtaThreads;
  const int g = p.heads[y], tid = threadIdx.x;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  const int n = sel_n(p, b, L, false);
  if (n == 0 || n >= L) return;  // nothing to select: the write phase alone
  const int64_t rid = (int64_t)g * p.B + b;
  const int nch = (L + kSelChunk - 1) / kSelChunk;
  const unsigned long long* cand = p.cand + (int64_t)g * p.T + off;
  const int T1 = __ldcg(p.row_info + rid * kRowInfo), above1 = __ldcg(p.row_info + rid * kRowInfo + 1);
  const int m = __ldcg(p.cand_count + rid);
  const bool in_smem = m <= kSelResolveCap;
  __syncthreads();  // the scratch may still be read for the previous item
  if (in_smem) {
    for (int j = tid; j < m; j += NT) {
      const unsigned long long e = __ldcg(cand + j);
      s_key[j] = (uint32_t)(e >> 32);
      s_chk[j] = (uint16_t)((uint32_t)e / kSelChunk);
    }
  }
  for (int q = tid; q < nch; q += NT) {
    s_gt[q] = 0;
    s_eq[q] = 0;
  }
  for (int i = tid; i < kSelHistBins; i += NT) p.hist[rid * kSelHistBins + i] = 0u;
  uint32_t prefix = (uint32_t)T1 << kSelHistShift, pmask = 0xffffffffu << kSelHistShift;
  int krem = n - above1;
#pragma unroll 1
  for (int d = 0; d < 2; ++d) {
    const int sh = d == 0 ? 10 : 0;
    const int nb = d == 0 ? 2048 : 1024;
    for (int i = tid; i < nb; i += NT) s_hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < m; j += NT) {
      const uint32_t kj = in_smem ? s_key[j] : (uint32_t)(__ldcg(cand + j) >> 32);
      if ((kj & pmask) == prefix) atomicAdd(&s_hist[(kj >> sh) & (nb - 1)], 1);
    }
    __syncthreads();
    // bins from the top: thread t takes per = nb / NT consecutive bins
    const int per = nb / NT;
    int cnt[8], sum = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cnt[u] = u < per ? s_hist[nb - 1 - (tid * per + u)] : 0;
      sum += cnt[u];
    }
    int total;
    int excl = block_exclusive_scan(sum, scratch, &total);
    if (excl < krem && krem <= excl + sum) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (u < per && excl < krem && krem <= excl + cnt[u]) {
          s_out[0] = nb - 1 - (tid * per + u);
          s_out[1] = excl;
          s_out[2] = cnt[u];
        }
        excl += cnt[u];
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_out[0] << sh;
    pmask |= (uint32_t)(nb - 1) << sh;
    krem -= s_out[1];
    const bool whole_bin = s_out[2] == krem;  // the same in every thread
    __syncthreads();
    if (whole_bin) break;
  }
  const int need_eq = krem;  // keys equal (masked) to the prefix that are taken, lowest positions first
  // candidates above / equal to the threshold, per chunk
  for (int j = tid; j < m; j += NT) {
    uint32_t kj;
    int q;
    if (in_smem) {
      kj = s_key[j];
      q = s_chk[j];
    } else {
      const unsigned long long e = __ldcg(cand + j);
      kj = (uint32_t)(e >> 32);
      q = (int)((uint32_t)e / kSelChunk);
    }
    const uint32_t mk = kj & pmask;
    if (mk > prefix) atomicAdd(&s_gt[q], 1);
    else if (mk == prefix) atomicAdd(&s_eq[q], 1);
  }
  __syncthreads();
  // offsets: thread t owns chunks [t * per, (t + 1) * per)
  const int per = (nch + NT - 1) / NT;
  const int q0 = min(nch, tid * per), q1 = min(nch, q0 + per);
  int sel_t = 0, eq_t = 0;
  for (int q = q0; q < q1; ++q) {
    sel_t += __ldcg(p.chunk_above + rid * p.max_chunks + q) + s_gt[q];
    eq_t += s_eq[q];
  }
  int tot_sel, tot_eq;
  int sel_before = block_exclusive_scan(sel_t, scratch, &tot_sel);
  int eq_before = block_exclusive_scan(eq_t, scratch, &tot_eq);
  for (int q = q0; q < q1; ++q) {
    p.chunk_info[(rid * p.max_chunks + q) * 2] = sel_before + min(need_eq, eq_before);
    p.chunk_info[(rid * p.max_chunks + q) * 2 + 1] = eq_before;
    sel_before += __ldcg(p.chunk_above + rid * p.max_chunks + q) + s_gt[q];
    eq_before += s_eq[q];
  }
  if (tid == 0) {
    p.row_info[rid * kRowInfo + 2] = (int)prefix;
    p.row_info[rid * kRowInfo + 3] = (int)pmask;
    p.row_info[rid * kRowInfo + 4] = need_eq;
  }
}

// ---------------------------------------------------------------------------- write phase
__device__ __forceinline__ void sel_write_item(const HistSelectParams& p, uint8_t* sm, int c, int y, int b) {
  int* scratch = reinterpret_cast<int*>(sm);  // [33]
  const int g = p.heads[y], tid = threadIdx.x;
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
  const float* row = p.scores + (int64_t)g * p.T + off;
  // the chunk's keys (warp w owns keys [i0 + w * 32 * kWriteK, ...), lane-consecutive loads)
  // and the row's threshold: all loads in flight together
  const int w0 = i0 + warp * 32 * kWriteK;
  uint32_t k[kWriteK];
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    const int i = w0 + r * 32 + lane;
    k[r] = i < i1 ? score_key(__ldcg(row + i)) : 0u;
  }
  const uint32_t KT = (uint32_t)__ldcg(p.row_info + rid * kRowInfo + 2);
  const uint32_t pmask = (uint32_t)__ldcg(p.row_info + rid * kRowInfo + 3);
  const int need_eq = __ldcg(p.row_info + rid * kRowInfo + 4);
  const int sel_chunk = __ldcg(p.chunk_info + (rid * p.max_chunks + c) * 2);
  const int eq_chunk = __ldcg(p.chunk_info + (rid * p.max_chunks + c) * 2 + 1);
  int ngt = 0, neq = 0;
#pragma unroll
  for (int r = 0; r < kWriteK; ++r) {
    const int i = w0 + r * 32 + lane;
    ngt += (i < i1 && (k[r] & pmask) > KT);
    neq += (i < i1 && (k[r] & pmask) == KT);
  }
  ngt = __reduce_add_sync(0xffffffffu, ngt);
  neq = __reduce_add_sync(0xffffffffu, neq);
  __syncthreads();  // the scratch may still be read for the previous item
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
    const bool gt = in && (k[r] & pmask) > KT;
    const bool eq = in && (k[r] & pmask) == KT;
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

// ---------------------------------------------------------------------------- kernels
// One kernel per phase: grid (max_chunks, listed heads, sequences); the resolve (1, heads, sequences).
__global__ void __launch_bounds__(kSelCtaThreads) select_hist_kernel(const HistSelectParams p) {
  grid_dep_wait();  // inputs come from the kernel before this one
  grid_dep_launch();
  __shared__ __align__(16) uint8_t sm[4 * kSelHistBins];
  sel_hist_item(p, sm, blockIdx.x, blockIdx.y, blockIdx.z);
}

__global__ void __launch_bounds__(kSelCtaThreads) select_chunk_kernel(const HistSelectParams p) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ __align__(16) uint8_t sm[256];
  sel_chunk_item(p, sm, blockIdx.x, blockIdx.y, blockIdx.z);
}

__global__ void __launch_bounds__(kSelCtaThreads) select_resolve_kernel(const HistSelectParams p) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ __align__(16) uint8_t sm[kSelSmem];
  sel_resolve_row(p, sm, blockIdx.y, blockIdx.z);
}

__global__ void __launch_bounds__(kSelCtaThreads) select_write_kernel(const HistSelectParams p) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ __align__(16) uint8_t sm[256];
  sel_write_item(p, sm, blockIdx.x, blockIdx.y, blockIdx.z);
}

}  // namespace aoh
