// Top-N_fac selection over precomputed scores, one thread-block cluster per row
// (FASA: Frequency-aware Sparse Attention, §2.B.1, keep the N_fac best tokens; the shared
// index of "Cómo funciona CLSA" is the same operation with k fixed).
//
// Same result as the chunked select (select_hist.cuh): the selection of a (sequence b,
// KV head g) row is {key > K_T} plus the lowest positions among {key == K_T}, n in all,
// written in ascending position order; keys are the order-preserving uint32 images of the
// fp32 scores.  For rows of at most kScMaxCluster x kScSlice positions the whole select
// runs on chip in one launch:
//   * the row is split into CL contiguous slices, one per CTA of the cluster; every thread
//     holds kScK keys of its slice in registers (warp w owns a run of 32 x kScK
//     consecutive positions, lane-interleaved), loaded once;
//   * MSB radix select with digits of 11, 11 and 10 bits: every CTA counts the keys that
//     match the prefix so far into a shared histogram and adds its non-zero bins into the
//     same digit's total of every peer (remote atomics), so that after one cluster barrier
//     every CTA holds the cluster's histogram and picks the same digit.  When the chosen
//     bin holds exactly the keys still needed, the remaining digits are skipped: every key
//     of the bin is taken, whatever its low bits;
//   * every CTA counts its keys above and inside the threshold and stores the two counts
//     in every peer; after one more barrier each CTA knows how many positions the slices
//     before it take, and its warps write their picks in order (ballots, one block scan).
// No workspace, no atomics in global memory, deterministic.
#pragma once

#include <cooperative_groups.h>

#include "device_common.cuh"

namespace aoh {

constexpr int kScThreads = 512;
constexpr int kScK = 16;                        // keys per thread
constexpr int kScSlice = kScThreads * kScK;     // positions per CTA (8192)
constexpr int kScMaxCluster = 16;
constexpr int kScBins = 2048;

struct ClusterSelectParams {
  const float* scores;           // [Hkv][T]
  const int32_t* offsets;        // [B + 1]
  const int32_t* lengths;        // [B] or null
  const int32_t* n_fac_per_seq;  // [B] or null
  int32_t* idx;                  // [B][Hkv][cap]
  int32_t* count;                // [B][Hkv]
  int32_t T, Hkv, n_fac, cap;
  uint8_t heads[kMaxHeads];      // KV head of blockIdx.y
};

__global__ void __launch_bounds__(kScThreads) select_cluster_kernel(const ClusterSelectParams p) {
  grid_dep_wait();  // the scores come from the kernel before this one
  grid_dep_launch();
  namespace cgs = cooperative_groups;
  __shared__ int tot[3][kScBins];  // cluster totals of each digit (filled by every CTA)
  __shared__ int lh[kScBins];      // this CTA's counts of the current digit
  __shared__ int scratch[33];
  __shared__ int s_pick[3];        // digit, keys in higher bins, keys in the digit's bin
  __shared__ int s_warp[2][kScThreads / 32];
  __shared__ int s_peer[kScMaxCluster][2];  // keys above / inside the threshold of every CTA
  cgs::cluster_group cluster = cgs::this_cluster();
  const int CL = (int)cluster.num_blocks(), rk = (int)cluster.block_rank();
  const int g = p.heads[blockIdx.y], b = blockIdx.z, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  int nf = p.n_fac_per_seq ? p.n_fac_per_seq[b] : p.n_fac;
  if (nf > p.cap) {
    if (rk == 0 && tid == 0) record_error(kCheckCount, b, nf, p.cap);
    nf = p.cap;
  }
  const int n = max(0, min(nf, L));
  int32_t* out = p.idx + ((int64_t)b * p.Hkv + g) * p.cap;
  if (rk == 0) {
    for (int j = n + tid; j < p.cap; j += kScThreads) out[j] = -1;
    if (tid == 0) p.count[(int64_t)b * p.Hkv + g] = n;
  }
  // this CTA's slice of the row (the host sizes the cluster so that it holds kScSlice at most)
  const int S = (L + CL - 1) / CL;
  const int a0 = min(L, rk * S), a1 = min(L, a0 + S);
  if (n == 0) return;  // n and L are the same for the whole cluster: no barrier is taken
  if (n >= L) {        // every position, in order
    for (int i = a0 + tid; i < a1; i += kScThreads) out[i] = i;
    return;
  }
  for (int j = tid; j < 3 * kScBins; j += kScThreads) (&tot[0][0])[j] = 0;
  for (int j = tid; j < kScBins; j += kScThreads) lh[j] = 0;
  cluster_arrive_release();  // the totals are zero before any peer adds into them

  // keys of this thread: positions w0 + r * 32 + lane, r < kScK
  const int w0 = a0 + warp * 32 * kScK;
  const int nv = max(0, min(a1 - w0, 32 * kScK));  // valid positions of this warp's run
  const float* row = p.scores + (int64_t)g * p.T + off;
  uint32_t k[kScK];
#pragma unroll
  for (int r = 0; r < kScK; ++r) k[r] = r * 32 + lane < nv ? score_key(__ldcg(row + w0 + r * 32 + lane)) : 0u;
  __syncthreads();  // lh is zero

  uint32_t prefix = 0u, pmask = 0u;
  int krem = n;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass < 2 ? kScBins : kScBins / 2;
#pragma unroll
    for (int r = 0; r < kScK; ++r)
      if (r * 32 + lane < nv && (k[r] & pmask) == prefix) atomicAdd(&lh[(k[r] >> sh) & (uint32_t)(nb - 1)], 1);
    __syncthreads();
    if (pass == 0) cluster_wait_acquire();  // every peer has zeroed its totals
    for (int j = tid; j < nb; j += kScThreads) {
      const int c = lh[j];
      if (c) {
        for (int q = 0; q < CL; ++q) atomicAdd(cluster.map_shared_rank(&tot[pass][j], q), c);
        lh[j] = 0;  // read only by this thread: ready for the next digit
      }
    }
    cluster.sync();  // every peer's counts are in tot[pass]
    // the bin holding the krem-th largest key: thread t takes nb / kScThreads bins from the top
    const int per = nb / kScThreads;
    int cnt[kScBins / kScThreads], sum = 0;
#pragma unroll
    for (int j = 0; j < kScBins / kScThreads; ++j) {
      cnt[j] = j < per ? tot[pass][nb - 1 - (tid * per + j)] : 0;
      sum += cnt[j];
    }
    int total;
    int above = block_exclusive_scan(sum, scratch, &total);
    if (above < krem && krem <= above + sum) {
#pragma unroll
      for (int j = 0; j < kScBins / kScThreads; ++j) {
        if (j < per && above < krem && krem <= above + cnt[j]) {
          s_pick[0] = nb - 1 - (tid * per + j);
          s_pick[1] = above;
          s_pick[2] = cnt[j];
        }
        above += cnt[j];
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_pick[0] << sh;
    pmask |= (uint32_t)(nb - 1) << sh;
    krem -= s_pick[1];
    const bool whole_bin = s_pick[2] == krem;  // the same in every CTA of the cluster
    __syncthreads();                            // s_pick is rewritten by the next digit
    if (whole_bin) break;
  }
  // threshold: keys whose masked value is above `prefix` are taken, and the first `krem`
  // (in position order) of those equal to it
  const int need_eq = krem;
  int gt = 0, eq = 0;
#pragma unroll
  for (int r = 0; r < kScK; ++r) {
    const bool in = r * 32 + lane < nv;
    const uint32_t m = k[r] & pmask;
    gt += in && m > prefix;
    eq += in && m == prefix;
  }
  gt = __reduce_add_sync(0xffffffffu, gt);
  eq = __reduce_add_sync(0xffffffffu, eq);
  if (lane == 0) {
    s_warp[0][warp] = gt;
    s_warp[1][warp] = eq;
  }
  __syncthreads();
  if (tid < CL) {
    int cg = 0, ce = 0;
    for (int w = 0; w < kScThreads / 32; ++w) {
      cg += s_warp[0][w];
      ce += s_warp[1][w];
    }
    int* dst = cluster.map_shared_rank(&s_peer[rk][0], tid);
    dst[0] = cg;
    dst[1] = ce;
  }
  cluster.sync();  // every CTA's counts are in s_peer; no remote access follows
  int sel_cta = 0, eq_cta = 0;
  for (int q = 0; q < rk; ++q) {
    sel_cta += s_peer[q][0];
    eq_cta += s_peer[q][1];
  }
  sel_cta += min(need_eq, eq_cta);  // equal keys taken before this slice
  int gt_before = 0, eq_before = eq_cta;
  for (int w = 0; w < warp; ++w) {
    gt_before += s_warp[0][w];
    eq_before += s_warp[1][w];
  }
  int sel_before = sel_cta + gt_before + (min(need_eq, eq_before) - min(need_eq, eq_cta));
#pragma unroll
  for (int r = 0; r < kScK; ++r) {
    const bool in = r * 32 + lane < nv;
    const uint32_t m = k[r] & pmask;
    const bool e = in && m == prefix;
    const unsigned be = __ballot_sync(0xffffffffu, e);
    const bool take = (in && m > prefix) || (e && eq_before + __popc(be & ((1u << lane) - 1u)) < need_eq);
    const unsigned bt = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int o = sel_before + __popc(bt & ((1u << lane) - 1u));
      if (o < n) out[o] = w0 + r * 32 + lane;  // o < n by construction; kept as a guard
    }
    sel_before += __popc(bt);
    eq_before += __popc(be);
  }
}

}  // namespace aoh
