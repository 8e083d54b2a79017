// Top-N_fac selection (FASA: Frequency-aware Sparse Attention, §2.B.1; the
// shared index of "Cómo funciona CLSA" is the same operation with k fixed).
//
// One thread-block cluster per (sequence b, KV head g).  The row's scores are
// split into CL contiguous slices, one per CTA, cached in shared memory as
// order-preserving uint32 keys.  An MSB-first radix select (4 digits of 8 bits)
// finds the n-th largest key K_T: each CTA builds a 256-bin histogram of the keys
// that still match the prefix, every CTA sums the CL histograms through
// distributed shared memory and picks the same digit.  Histograms are double
// buffered so one cluster barrier per digit suffices.  The selection is then
// {key > K_T} plus the first (n - #{key > K_T}) positions with key == K_T in
// position order, which is exactly "score descending, lower position first".
// An ordered compaction (block scans inside a CTA, a cluster-wide prefix over the
// CTA totals) writes the positions in ascending order.  Deterministic.
#pragma once

#include <cooperative_groups.h>

#include "device_common.cuh"

namespace aoh {

namespace cg = cooperative_groups;

constexpr int kSelThreads = 512;

struct SelectParams {
  const float* scores;            // [Hkv][T]
  const int32_t* offsets;         // [B + 1]
  const int32_t* n_fac_per_seq;   // [B] or null
  int32_t* idx;                   // [B][Hkv][cap]
  int32_t* count;                 // [B][Hkv]
  int32_t T, Hkv, n_fac, cap;
  int32_t chunk;                  // positions per CTA slice
  int32_t keys_in_smem;           // 1: slice cached in dynamic shared memory
  uint8_t heads[kMaxHeads];
};


__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(const SelectParams p) {
  extern __shared__ __align__(16) uint32_t skeys[];
  __shared__ int hist[2][256];
  __shared__ int scan_scratch[33];
  __shared__ int s_bin, s_above;
  __shared__ int s_cnt[2];            // this CTA's (#eq, #gt)
  __shared__ int s_eq_before, s_sel_before;

  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int r = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const int b = blockIdx.z;
  const int g = p.heads[blockIdx.y];
  const int off = p.offsets[b];
  const int L = p.offsets[b + 1] - off;
  int nf = p.n_fac_per_seq ? p.n_fac_per_seq[b] : p.n_fac;
  if (nf > p.cap) {
    if (r == 0 && tid == 0) record_error(kCheckCount, b, nf, p.cap);
    nf = p.cap;
  }
  const int n = max(0, min(nf, L));
  int32_t* out = p.idx + ((int64_t)b * p.Hkv + g) * p.cap;
  const float* row = p.scores + (int64_t)g * p.T + off;
  const int lo = min(L, r * p.chunk);
  const int hi = min(L, lo + p.chunk);

  // padding of the unused tail of the row, spread over the cluster
  for (int j = n + r * kSelThreads + tid; j < p.cap; j += CL * kSelThreads) out[j] = -1;
  if (r == 0 && tid == 0) p.count[(int64_t)b * p.Hkv + g] = n;
  if (n == 0) return;               // uniform over the cluster: no barrier taken
  if (n == L) {                     // N_fac >= L: every position, in order
    for (int j = lo + tid; j < hi; j += kSelThreads) out[j] = j;
    return;
  }

  if (p.keys_in_smem) {
    for (int i = lo + tid; i < hi; i += kSelThreads) skeys[i - lo] = score_key(row[i]);
  }
  auto key_at = [&](int i) -> uint32_t {  // i in [lo, hi)
    return p.keys_in_smem ? skeys[i - lo] : score_key(__ldcg(row + i));
  };

  uint32_t prefix = 0u, pmask = 0u;
  int krem = n;  // rank of the threshold among keys matching the prefix (1-based from the top)
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    int* h = hist[pass & 1];
    if (tid < 256) h[tid] = 0;
    __syncthreads();
    if (p.keys_in_smem) {
      // four keys per lane from shared memory; the first digit (sign + exponent) is shared by
      // most keys and counted with warp aggregation, later digits directly
      for (int b0 = (tid & ~31) * 4; b0 < hi - lo; b0 += kSelThreads * 4) {  // warp-uniform
        const int i0 = b0 + 4 * (tid & 31);  // i0 + 3 < chunk: inside the keys region
        const uint4 k4 = *reinterpret_cast<const uint4*>(skeys + i0);
        const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool in = (i0 + j < hi - lo) && ((kk[j] & pmask) == prefix);
          const int bin = in ? (int)((kk[j] >> shift) & 255u) : -1;
          if (pass == 0) {
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (bin >= 0 && (tid & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
          } else if (in) {
            atomicAdd(&h[bin], 1);
          }
        }
      }
    } else {
      // scores re-read from L2: warp-aggregated counts
      for (int base = lo + (tid & ~31); base < hi; base += kSelThreads) {
        const int i = base + (tid & 31);
        int bin = -1;
        if (i < hi) {
          const uint32_t k = key_at(i);
          if ((k & pmask) == prefix) bin = (int)((k >> shift) & 255u);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin >= 0 && (tid & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], __popc(peers));
      }
    }
    cluster.sync();
    // cluster-wide total of the bin that this thread scans, bins taken from the top down
    int tot = 0;
    if (tid < 256) {
      const int bin = 255 - tid;
      int v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = (q < CL) ? cluster.map_shared_rank(h, q)[bin] : 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) tot += v[q];
    }
    int total;
    const int above = block_exclusive_scan(tot, scan_scratch, &total);
    if (tid < 256 && above < krem && krem <= above + tot) {
      s_bin = 255 - tid;
      s_above = above;
    }
    __syncthreads();
    prefix |= (uint32_t)s_bin << shift;
    pmask |= 255u << shift;
    krem -= s_above;
    __syncthreads();
  }
  const uint32_t KT = prefix;
  const int need_eq = krem;  // how many positions with key == KT are taken (lowest first)

  // ---- ordered compaction
  const int m = hi - lo;
  const int run = (m + kSelThreads - 1) / kSelThreads;
  const int a0 = lo + min(m, tid * run);
  const int a1 = lo + min(m, (tid + 1) * run);
  int n_eq = 0, n_gt = 0;
  for (int i = a0; i < a1; ++i) {
    const uint32_t k = key_at(i);
    n_gt += k > KT;
    n_eq += k == KT;
  }
  int eq_cta, gt_cta;
  const int eq_excl = block_exclusive_scan(n_eq, scan_scratch, &eq_cta);
  block_exclusive_scan(n_gt, scan_scratch, &gt_cta);
  if (tid == 0) {
    s_cnt[0] = eq_cta;
    s_cnt[1] = gt_cta;
  }
  cluster.sync();
  if (tid == 0) {
    int eq_before = 0, sel_before = 0;
    for (int q = 0; q < r; ++q) {
      const int* c = cluster.map_shared_rank(s_cnt, q);
      const int eqq = c[0], gtq = c[1];
      sel_before += gtq + max(0, min(need_eq - eq_before, eqq));
      eq_before += eqq;
    }
    s_eq_before = eq_before;
    s_sel_before = sel_before;
  }
  __syncthreads();
  cluster_arrive_release();  // this CTA is done reading its peers' shared memory
  const int eq_base = s_eq_before + eq_excl;
  int n_sel = 0;
  {
    int seen = 0;
    for (int i = a0; i < a1; ++i) {
      const uint32_t k = key_at(i);
      if (k > KT) {
        ++n_sel;
      } else if (k == KT) {
        n_sel += (eq_base + seen < need_eq);
        ++seen;
      }
    }
  }
  int sel_cta;
  int pos = s_sel_before + block_exclusive_scan(n_sel, scan_scratch, &sel_cta);
  {
    int seen = 0;
    for (int i = a0; i < a1; ++i) {
      const uint32_t k = key_at(i);
      bool take = false;
      if (k > KT) {
        take = true;
      } else if (k == KT) {
        take = (eq_base + seen < need_eq);
        ++seen;
      }
      if (take && pos < n) out[pos++] = i;  // pos < n holds by construction; kept as a guard
    }
  }
  cluster_wait_acquire();  // peers may still read s_cnt until they have all arrived
}

}  // namespace aoh
