// Fused decode step of one SPARSE (sequence, KV head) row in one thread-block
// cluster: importance scan -> top-N_fac -> focused attention -> combine.
//
// FASA: Frequency-aware Sparse Attention, §2.B.1 (importance from the dominant
// chunks, keep the N_fac best) and §2.B.2 (full-dimension attention over the
// kept tokens at their original positions); the shared-index stack of "Cómo
// funciona CLSA" is the same row with every chunk scored and NQ = n_layers * G.
//
// The row's L positions are cut into CL contiguous slices, one per CTA.
//  1. scan:    each CTA streams the score rows of its slice (packed dominant
//              columns, or K in place): every warp runs its own cp.async ring of
//              16-byte row segments, 16 in flight per lane, and takes the fp32 dots
//              with the group-summed query (the same arithmetic as the stand-alone
//              scan kernel); the scores stay in shared memory as order-preserving
//              uint32 keys;
//  2. select:  MSB radix select of the n-th largest key over the cluster, up to 4
//              digits of 8 bits (histograms summed through distributed shared memory,
//              one cluster barrier per digit; it stops at the first digit whose chosen
//              bin is exactly what is left); ties broken toward lower positions by an
//              ordered compaction that also writes the index (ascending) to global memory;
//  3. attend:  every CTA gathers the K / V rows of the positions it selected from
//              its own slice (cp.async into tiles at a 2*d+16-byte row pitch) and
//              runs the online-softmax contraction on tensor cores (tokens on M,
//              query rows on N, P as hi + lo bf16 parts); the 8 warps split the
//              tokens, the query n-tiles and 2-4 parts of the head dimension of
//              the PV product;
//  4. combine: the CL partial (m, l, acc) states are merged through distributed
//              shared memory, each CTA writing 1/CL of the outputs.
// Nothing but the index and the outputs goes to global memory; no global
// scratch, no second launch.  Select-only mode takes the keys from scores that the
// stand-alone scan wrote and stops after 2 (fewer rows than SMs, each spread over a
// cluster's shared memory).  DENSE / STREAM heads may ride in the same launch: their
// clusters skip 1-2 and attend over their range (the whole AoH step in one launch).
#pragma once

#include <cooperative_groups.h>

#include "device_common.cuh"

namespace aoh {

namespace cgs = cooperative_groups;

constexpr int kSrThreads = 256;  // 8 warps
constexpr int kSrTS = 32;        // tokens per attention stage
constexpr int kSrMaxStages = 8;  // ring stages (run-time count, from the shared memory left)
constexpr int kSrMaxCluster = 16;
constexpr int kSrMaxRun = 64;    // keys per thread in the compaction: slice <= 256 * 64
constexpr int kScanU = 4;        // scan: rows per lane per cp.async group
constexpr int kScanDepth = 4;    // scan: groups in flight per warp (ring = 8 warps x 8 KB)
constexpr int kSrRingMin = 8 * kScanDepth * kScanU * 512;  // 64 KB

struct RowParams {
  const uint16_t* q_score;   // [B][Hq][D]: the query that scores (group-summed)
  const uint16_t* q_attn;    // [n_layers][B][Hq][D]: query rows of the attention
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* offsets;    // [B + 1]
  const int32_t* lengths;    // [B] or null (sequences fill their regions)
  const uint16_t* score_src; // packed k_dom or K
  int64_t srow_stride_tok, srow_stride_head;
  int32_t srow_len;          // elements per score row: 16, 32, 64 or 128 (k_dom cols, or D in place)
  int32_t packed;            // 1: k_dom rows; 0: K rows with q masked to the dominant dims
  const int32_t* idom;       // [Hkv][n_dom]; null = every chunk
  int32_t n_dom;
  const int32_t* n_fac_per_seq;
  int32_t n_fac, cap;
  int32_t* idx_out;          // [B][Hkv][cap]
  int32_t* count_out;        // [B][Hkv]
  float* out;                // [n_layers][B][Hq][D]
  int64_t stride_tok, stride_head;
  int32_t T, B, Hq, Hkv, G, NQ;
  int32_t keys_bytes;        // dynamic shared memory before the ring
  int32_t ring_bytes;        // ring region (scan rings, then attention stages); >= kSrRingMin
  float scale_log2;
  uint8_t heads[kMaxHeads];
  uint8_t slot[kMaxHeads];   // head slot of every KV head in K / V and in the score rows
  uint8_t roles[kMaxHeads];  // 0 SPARSE (scan, select, attend); 1 DENSE / 2 STREAM: attend over the range
  int32_t sink, window;      // the STREAM range: [0, min(sink, L)) U [max(sink, L - window), L)
  const float* scores_in;    // select-only form: the keys come from these fp32 scores [Hkv][T]
};

// Attention tiles: gathered K / V rows are copied as 16-byte cp.async segments into rows
// of pitch 2*D + 16 bytes, so the 8 rows an ldmatrix reads sit in 8 different 16-byte
// bank groups.
template <int D>
struct AttTile {
  static constexpr int kPitch = 2 * D + 16;
  static constexpr int kTile = kSrTS * kPitch;  // one of K or V per stage
  static constexpr int kStage = 2 * kTile;
};

// SO: the select-only form (keys loaded from p.scores_in, no scan, stops once the index is
// written: no attention, no outputs).
template <int D, int NT, bool SO>
__global__ void __launch_bounds__(kSrThreads) sparse_row_kernel(const __grid_constant__ RowParams p) {
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(NT == 1 || NT == 2 || NT == 4, "n-tiles");
  constexpr int KS = D / 16;          // k-steps of QK
  constexpr int DP = (NT == 4) ? 2 : 4;  // parts of the head dimension in the PV product
  constexpr int TG = 8 / (NT * DP);      // token groups (warps sharing an n-tile and a part)
  constexpr int KH = KS / DP;            // PV m-tiles per part
  constexpr int SUB = kSrTS / 16;     // 16-token sub-tiles per stage
  constexpr int NQP = NT * 8;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ int lhb[2][256];  // this CTA's histogram of digit p in lhb[p & 1] (one cleared per digit)
  __shared__ int tot[2][256];  // cluster totals of digits 0-2 (every CTA adds its counts here)
  __shared__ int scan_scratch[33];
  __shared__ float qt[128];
  __shared__ int s_bin, s_above, s_eq_before, s_sel_before, s_up;
  __shared__ int s_gt[kSrMaxCluster], s_eq[kSrMaxCluster], s_eq_all;

  cgs::cluster_group cluster = cgs::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rk = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.z;
  const int g = p.heads[blockIdx.y];
  int off;
  const int L = seq_length(p.offsets, p.lengths, b, false, &off);
  int nf = p.n_fac_per_seq ? p.n_fac_per_seq[b] : p.n_fac;
  if (nf > p.cap) {
    if (rk == 0 && tid == 0) record_error(kCheckCount, b, nf, p.cap);
    nf = p.cap;
  }
  const int n = max(0, min(nf, L));
  // a window head (DENSE or STREAM role, AoH summary Metodología §4) attends over its range,
  // split evenly across the cluster: no scan, no select, no index written
  const int role = p.roles[g];
  int wra = 0, wrb = 0;
  if (role == 1) {
    wra = L;
    wrb = L;
  } else if (role == 2) {
    wra = min(p.sink, L);
    wrb = max(wra, L - p.window);
  }
  const int nwin = wra + (L - wrb);
  int32_t* idx_row = p.idx_out + ((int64_t)b * p.Hkv + g) * p.cap;
  if (role == 0) {
    for (int j = n + rk * kSrThreads + tid; j < p.cap; j += CL * kSrThreads) idx_row[j] = -1;
    if (rk == 0 && tid == 0) p.count_out[(int64_t)b * p.Hkv + g] = n;
  }
  if ((role == 0 ? n : nwin) == 0) {  // uniform over the cluster: zero rows, no barrier taken
    if (rk == 0 && !SO) {
      for (int e = tid; e < p.NQ * D; e += kSrThreads) {
        const int qr = e / D, l = qr / p.G, h = g * p.G + qr % p.G;
        p.out[(((int64_t)l * p.B + b) * p.Hq + h) * D + e % D] = 0.f;
      }
    }
    return;
  }

  if (tid < kSrMaxCluster) {
    s_gt[tid] = 0;
    s_eq[tid] = 0;
  }
  // the dynamic region is used from a 1 KB boundary (the host adds 1 KB of slack)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int slice = (((L + CL - 1) / CL) + 3) & ~3;
  const int lo = min(L, rk * slice), hi = min(L, lo + slice);
  const int m = hi - lo;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
  int* plist = reinterpret_cast<int*>(smem);  // selected positions replace the keys
  int nloc;

  // The select's totals are filled by every CTA of the cluster: zero them, then arrive on a
  // cluster barrier that is waited on only before the first remote add (the scan runs in between).
  if (role == 0 && n < L) {
    lhb[0][tid] = 0;
    lhb[1][tid] = 0;
    tot[0][tid] = 0;
    tot[1][tid] = 0;
    if (tid == 0) s_up = 0;
    __syncthreads();
    cluster_arrive_release();
  }
  if (role == 0 && n < L) {
    // =============================================================== 1. scan
    if constexpr (SO) {
      // the scores were computed by the stand-alone scan: load them as keys, eight loads
      // in flight per thread
      const float* srow = p.scores_in + (int64_t)g * p.T + off + lo;
      for (int i0 = 0; i0 < m; i0 += 8 * kSrThreads) {
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kSrThreads + tid;
          f[u] = i < m ? __ldcg(srow + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * kSrThreads + tid;
          if (i < m) keys[i] = score_key(f[u]);
        }
      }
      __syncthreads();
    } else {
      // Each warp streams a contiguous run of the slice's rows through its own cp.async
      // ring: S lanes share a row (16 bytes each), kScanU rows per lane per group,
      // kScanDepth groups in flight; the first groups are issued before the group-summed
      // query is built (its loads then overlap theirs).  A lane reads back only the bytes it
      // copied, so the ring needs no barrier; the dot and its shuffle reduction match the
      // stand-alone scan kernel term for term (same fp32 scores, same keys).
      const int S = p.srow_len >> 3;  // 2, 4, 8 or 16
      const int seg = lane & (S - 1);
      const int rpw = 32 / S;
      const int per_warp = (m + 7) / 8;
      const int wr0 = min(m, warp * per_warp), wr1 = min(m, wr0 + per_warp);
      const int grows = rpw * kScanU;
      const int nb = (wr1 - wr0 + grows - 1) / grows;
      const uint32_t wring = smem_u32(smem + p.keys_bytes) + warp * (kScanDepth * kScanU * 512) + lane * 16;
      const uint16_t* src0 = p.score_src + (int64_t)p.slot[g] * p.srow_stride_head + (int64_t)(off + lo) * p.srow_stride_tok + seg * 8;
      auto issue = [&](int k) {
        const uint32_t slot = wring + (k % kScanDepth) * (kScanU * 512);
#pragma unroll
        for (int u = 0; u < kScanU; ++u) {
          const int r = wr0 + k * grows + u * rpw + lane / S;
          const bool ok = r < wr1;
          cp_async_16(slot + u * 512, src0 + (int64_t)(ok ? r : wr0) * p.srow_stride_tok, ok);
        }
      };
#pragma unroll
      for (int k = 0; k < kScanDepth - 1; ++k) {
        if (k < nb) issue(k);
        cp_async_commit();
      }
      if (tid < p.srow_len) {
        const int C = D / 2;
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
          const uint16_t* qb = p.q_score + ((int64_t)b * p.Hq + (int64_t)g * p.G) * D + dim;
          for (int h0 = 0; h0 < p.G; h0 += 8) {  // eight loads in flight, summed in head order
            float qv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              qv[u] = (h0 + u < p.G) ? __uint_as_float((uint32_t)qb[(int64_t)(h0 + u) * D] << 16) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) acc += qv[u];
          }
        }
        qt[tid] = acc;
      }
      __syncthreads();
      float qs[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) qs[i] = qt[seg * 8 + i];
      for (int k = 0; k < nb; ++k) {
        if (k + kScanDepth - 1 < nb) issue(k + kScanDepth - 1);
        cp_async_commit();
        cp_async_wait<kScanDepth - 1>();
        const uint8_t* slot = smem + p.keys_bytes + warp * (kScanDepth * kScanU * 512) + lane * 16 +
                              (k % kScanDepth) * (kScanU * 512);
#pragma unroll
        for (int u = 0; u < kScanU; ++u) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(slot + u * 512);
          float sc = dot8(v4, qs);
          for (int o = S >> 1; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
          const int r = wr0 + k * grows + u * rpw + lane / S;
          if (seg == 0 && r < wr1) keys[r] = score_key(sc);
        }
      }
      cp_async_wait<0>();
      __syncthreads();
    }
    // =============================================================== 2. select
    // 4-digit MSB radix select over the cluster.  Digits 0-2: every CTA adds its non-zero
    // counts into each peer's total (remote atomics), one cluster barrier, then the digit is
    // picked from the local total.  Digit 3: every CTA reads each peer's last histogram, which
    // also gives each peer's number of keys above the threshold (s_gt) and equal to it (s_eq),
    // so the compaction needs no further exchange.  After digit 0 the keys sharing the chosen
    // first digit are compacted; digits 1-3 count only those.  When a digit's chosen bin holds
    // exactly the keys still needed, the remaining digits are skipped.
    cluster_wait_acquire();  // peers have zeroed their totals
    uint32_t* cand = reinterpret_cast<uint32_t*>(smem + p.keys_bytes);  // free region during the select
    uint32_t prefix = 0u, pmask = 0u;
    int krem = n;
    int ncand = 0;
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      int* lh = lhb[pass & 1];
      // the buffer of the next digit held digit pass - 1, whose readers passed the barrier
      // that ended that digit
      if (pass == 1 || pass == 2) lhb[(pass + 1) & 1][tid] = 0;
      if (pass == 0) {
        // the first digit (sign and exponent): plain shared-memory atomics (same-address
        // updates of one warp are combined by the hardware; faster here than aggregating
        // them with match.any)
        for (int b0 = warp * 128; b0 < m; b0 += 8 * 128) {
          const int i0 = b0 + 4 * lane;  // i0 + 3 < slice: inside the keys region
          const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i0);
          const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (i0 + j < m) atomicAdd(&lh[kk[j] >> 24], 1);
        }
      } else {
        // digits 1-3: over the compacted candidates, or over all keys when they did not fit
        const uint32_t* src = ncand >= 0 ? cand : keys;
        const int cnt = ncand >= 0 ? ncand : m;
        for (int b0 = warp * 128; b0 < cnt; b0 += 8 * 128) {
          const int i0 = b0 + 4 * lane;  // i0 + 3 inside the region (4 entries of slack)
          const uint4 k4 = *reinterpret_cast<const uint4*>(src + i0);
          const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (i0 + j < cnt && (kk[j] & pmask) == prefix) atomicAdd(&lh[(kk[j] >> shift) & 255u], 1);
        }
      }
      __syncthreads();
      const int bin = 255 - tid;  // the scan below runs from the top bin down
      int total_bin;
      int v[kSrMaxCluster];
      if (pass < 3) {
        const int c = lh[tid];
        if (c) {
          for (int q = 0; q < CL; ++q) atomicAdd(cluster.map_shared_rank(&tot[pass & 1][tid], q), c);
        }
        tot[(pass + 1) & 1][tid] = 0;  // peers add into it only after the barrier below
        cluster.sync();
        total_bin = tot[pass & 1][bin];
      } else {
        cluster.sync();  // every peer's last-digit histogram is complete
#pragma unroll
        for (int q = 0; q < kSrMaxCluster; ++q) v[q] = (q < CL) ? cluster.map_shared_rank(lh, q)[bin] : 0;
        total_bin = 0;
#pragma unroll
        for (int q = 0; q < kSrMaxCluster; ++q) total_bin += v[q];
      }
      // exclusive prefix over tid (bins from the top): warp scan, then the warp totals
      int x = total_bin;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane == 31) scan_scratch[warp] = x;
      __syncthreads();
      int above = x - total_bin;
      for (int w2 = 0; w2 < warp; ++w2) above += scan_scratch[w2];
      if (above < krem && krem <= above + total_bin) {
        s_bin = bin;
        s_above = above;
      }
      __syncthreads();
      const int sb = s_bin;
      if (pass < 3) {
        // this CTA's keys above the threshold decided by this digit
        const int w = __reduce_add_sync(0xffffffffu, bin > sb ? lh[bin] : 0);
        if (lane == 0 && w) atomicAdd(&s_up, w);
      } else {
#pragma unroll
        for (int q = 0; q < kSrMaxCluster; ++q) {
          if (q < CL) {
            const int w = __reduce_add_sync(0xffffffffu, bin > sb ? v[q] : 0);
            if (lane == 0 && w) atomicAdd(&s_gt[q], w);
          }
        }
        if (bin == sb) {
#pragma unroll
          for (int q = 0; q < kSrMaxCluster; ++q)
            if (q < CL) s_eq[q] = v[q];
        }
        if (tid < CL) atomicAdd(&s_gt[tid], *cluster.map_shared_rank(&s_up, tid));
      }
      // candidates of digits 1-3: the keys whose first digit is the chosen one, when they fit
      // the candidate region (this CTA's count of them is its own histogram's bin)
      const int n_sb = lh[sb];  // this CTA's keys in the chosen bin
      const bool compact = pass == 0 && n_sb <= p.ring_bytes / 4 - 4;
      if (compact) {
        // every warp counts its candidates (ballots), then writes them from its own offset
        // (the counts of the lower warps): no shared counter
        int wcnt = 0;
        for (int b0 = warp * 128; b0 < m; b0 += 8 * 128) {
          const int i0 = b0 + 4 * lane;
          const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i0);
          const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) wcnt += __popc(__ballot_sync(0xffffffffu, (i0 + j < m) && (int)(kk[j] >> 24) == sb));
        }
        if (lane == 0) scan_scratch[warp] = wcnt;
        __syncthreads();
        int wbase = 0;
        for (int w2 = 0; w2 < warp; ++w2) wbase += scan_scratch[w2];
        for (int b0 = warp * 128; b0 < m; b0 += 8 * 128) {
          const int i0 = b0 + 4 * lane;
          const uint4 k4 = *reinterpret_cast<const uint4*>(keys + i0);
          const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool hit = (i0 + j < m) && (int)(kk[j] >> 24) == sb;
            const unsigned bal = __ballot_sync(0xffffffffu, hit);
            if (hit) cand[wbase + __popc(bal & ((1u << lane) - 1u))] = kk[j];
            wbase += __popc(bal);
          }
        }
      }
      prefix |= (uint32_t)sb << shift;
      pmask |= 255u << shift;
      krem -= s_above;
      __syncthreads();
      if (pass == 0) ncand = compact ? n_sb : -1;
      // The chosen bin holds exactly the keys still needed (the same decision in every CTA):
      // it is taken whole, whatever its lower digits, and keys are compared masked.  Every
      // CTA's count above (s_up, final once the barrier below is passed) and its count in the
      // bin are what the compaction needs; neither is written again.
      if (pass < 3 && tot[pass & 1][sb] == krem) {
        cluster.sync();
        if (tid < CL) {
          s_gt[tid] = *cluster.map_shared_rank(&s_up, tid);
          s_eq[tid] = cluster.map_shared_rank(lhb[pass & 1], tid)[sb];
        }
        __syncthreads();
        break;
      }
    }
    const uint32_t KT = prefix;  // with pmask: keys are taken when (key & pmask) is above KT
    const int need_eq = krem;

    // ---- ordered compaction: positions in ascending order, lower position first among equals
    if (tid == 0) {
      int eq_before = 0, sel_before = 0, eq_all = 0;
      for (int q = 0; q < CL; ++q) {
        if (q < rk) {
          sel_before += s_gt[q] + max(0, min(need_eq - eq_before, s_eq[q]));
          eq_before += s_eq[q];
        }
        eq_all += s_eq[q];
      }
      s_eq_before = eq_before;
      s_sel_before = sel_before;
      s_eq_all = eq_all;
    }
    __syncthreads();
    const int run = (m + kSrThreads - 1) / kSrThreads;  // <= kSrMaxRun (host guarantees)
    const int a0 = min(m, tid * run), a1 = min(m, (tid + 1) * run);
    const int len = a1 - a0;
    // One pass over this thread's run of keys, in a lane-skewed order so that the 32 lanes
    // of a warp read 32 different banks: bit i of gtm / eqm marks key a0 + i above / equal
    // to the threshold.
    uint64_t gtm = 0ull, eqm = 0ull;
    if (len > 0) {
      int e = lane % len;
      for (int j = 0; j < len; ++j) {
        const uint32_t k = keys[a0 + e];
        gtm |= (uint64_t)((k & pmask) > KT) << e;
        eqm |= (uint64_t)((k & pmask) == KT) << e;
        if (++e == len) e = 0;
      }
    }
    const int n_eq = __popcll(eqm);
    int eq_excl = 0;
    if (s_eq_all > need_eq) {  // more keys equal the threshold than are taken: rank them
      int eq_cta;
      eq_excl = block_exclusive_scan(n_eq, scan_scratch, &eq_cta);
    }
    // this thread takes the lowest max(0, need_eq - equal keys before it) of its equal keys
    const int take_eq = min(n_eq, max(0, need_eq - (s_eq_before + eq_excl)));
    uint64_t take = gtm;
    if (take_eq == n_eq) {
      take |= eqm;
    } else {
      uint64_t rest = eqm;
      for (int i = 0; i < take_eq; ++i) {
        take |= rest & (~rest + 1ull);
        rest &= rest - 1ull;
      }
    }
    const int n_sel = __popcll(take);
    int sel_cta;
    const int my = block_exclusive_scan(n_sel, scan_scratch, &sel_cta);  // ends with a barrier
    {
      int o = my;
      const int gbase = s_sel_before;
      while (take) {
        const int bit = __ffsll((long long)take) - 1;
        take &= take - 1;
        const int pos = lo + a0 + bit;
        plist[o] = pos;
        if (gbase + o < n) idx_row[gbase + o] = pos;
        ++o;
      }
    }
    nloc = sel_cta;
  } else if (role == 0) {
    // N_fac >= L: every position of the slice, in order
    for (int i = tid; i < m; i += kSrThreads) {
      plist[i] = lo + i;
      idx_row[lo + i] = lo + i;
    }
    nloc = m;
  } else {
    // a window head: this CTA's share of the range (at most ceil(L / CL) <= slice entries)
    const int per = (nwin + CL - 1) / CL;
    const int j0 = min(nwin, rk * per), j1 = min(nwin, j0 + per);
    for (int i = tid; i < j1 - j0; i += kSrThreads) {
      const int j = j0 + i;
      plist[i] = j < wra ? j : wrb + (j - wra);
    }
    nloc = j1 - j0;
  }
  __syncthreads();
  if constexpr (SO) {  // the index is written; peers may still read this CTA's counts
    cluster.sync();
    return;
  }

  // =============================================================== 3. attend
  // warp = (token group, n-tile, part of the head dimension)
  const int dp = warp % DP, nt = (warp / DP) % NT, tg = warp / (DP * NT);
  float acc[KH][4];
#pragma unroll
  for (int i = 0; i < KH; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  uint8_t* stage_mem = smem + p.keys_bytes;
  const uint32_t sbase = smem_u32(stage_mem);
  const uint16_t* kbase = p.k + (int64_t)off * p.stride_tok + (int64_t)p.slot[g] * p.stride_head;
  const uint16_t* vbase = p.v + (int64_t)off * p.stride_tok + (int64_t)p.slot[g] * p.stride_head;
  const int nstages = (nloc + kSrTS - 1) / kSrTS;
  const int nsa = min(kSrMaxStages, p.ring_bytes / AttTile<D>::kStage);
  // every thread copies 16-byte chunks of the stage's K and V rows (cp.async); entries past
  // the list repeat its first position, so every row of a tile holds finite data
  auto issue_att = [&](int st) {
    if (st < nstages) {
      const uint32_t kt = sbase + (st % nsa) * AttTile<D>::kStage;
      const uint32_t vt = kt + AttTile<D>::kTile;
      constexpr int CPR = D / 8;
#pragma unroll
      for (int c = tid; c < kSrTS * CPR; c += kSrThreads) {
        const int r = c / CPR, ch = c % CPR;
        const int jj = st * kSrTS + r;
        const int pos = plist[jj < nloc ? jj : 0];
        const int64_t eo = (int64_t)pos * p.stride_tok + ch * 8;
        const uint32_t so = r * AttTile<D>::kPitch + ch * 16;
        cp_async_16(kt + so, kbase + eo, true);
        cp_async_16(vt + so, vbase + eo, true);
      }
    }
    cp_async_commit();
  };
  for (int s0 = 0; s0 < nsa - 1; ++s0) issue_att(s0);
  uint32_t bq[KS][2];
  {
    const int qr = nt * 8 + (lane >> 2);
    if (qr < p.NQ) {
      const int l = qr / p.G, h = g * p.G + qr % p.G;
      const uint16_t* qp = p.q_attn + (((int64_t)l * p.B + b) * p.Hq + h) * D + 2 * (lane & 3);
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
  for (int st = 0; st < nstages; ++st) {
    cp_async_wait_n(nsa - 2);
    __syncthreads();
    issue_att(st + nsa - 1);
    const uint32_t kt = sbase + (st % nsa) * AttTile<D>::kStage;
    const uint32_t vt = kt + AttTile<D>::kTile;
#pragma unroll
    for (int u = 0; u < SUB; ++u) {
      if ((st * SUB + u) % TG != tg) continue;
      const int nv = nloc - (st * kSrTS + u * 16);
      if (nv <= 0) continue;
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int r = u * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int dsel = (lane >> 4) * 8;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a[4];
          ldsm_x4(a, kt + r * AttTile<D>::kPitch + (ks * 16 + dsel) * 2);
          mma_16816(s4, a, bq[ks][0], bq[ks][1]);
        }
      }
      const int ta = lane >> 2, tb2 = ta + 8;
      const float x0 = ta < nv ? s4[0] * p.scale_log2 : -INFINITY;
      const float x1 = ta < nv ? s4[1] * p.scale_log2 : -INFINITY;
      const float x2 = tb2 < nv ? s4[2] * p.scale_log2 : -INFINITY;
      const float x3 = tb2 < nv ? s4[3] * p.scale_log2 : -INFINITY;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
      const float p0 = exp2f(x0 - mn0), p1 = exp2f(x1 - mn1);
      const float p2 = exp2f(x2 - mn0), p3 = exp2f(x3 - mn1);
      l0 = l0 * al0 + p0 + p2;
      l1 = l1 * al1 + p1 + p3;
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int i2 = 0; i2 < KH; ++i2) {
        acc[i2][0] *= al0;
        acc[i2][1] *= al1;
        acc[i2][2] *= al0;
        acc[i2][3] *= al1;
      }
      const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
      const uint32_t l01 = pack_bf16x2(p0 - bf16lo(h01), p1 - bf16hi(h01));
      const uint32_t l23 = pack_bf16x2(p2 - bf16lo(h23), p3 - bf16hi(h23));
      const uint32_t pb0 = movmatrix_trans(h01), pb1 = movmatrix_trans(h23);
      const uint32_t pl0 = movmatrix_trans(l01), pl1 = movmatrix_trans(l23);
      {
        const int r = u * 16 + (lane & 7) + (lane >> 4) * 8;
        const int dsel = ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int mt = 0; mt < KH; ++mt) {
          uint32_t a[4];
          ldsm_x4_trans(a, vt + r * AttTile<D>::kPitch + ((dp * KH + mt) * 16 + dsel) * 2);
          mma_16816(acc[mt], a, pb0, pb1);
          mma_16816(acc[mt], a, pl0, pl1);
        }
      }
    }
  }
  cp_async_wait<0>();
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  __syncthreads();  // stage buffers are free

  // ---- merge the warps of this CTA: red_ml [8][8][2], red_acc [8][8][D/DP]; CTA state after
  constexpr int DW = D / DP;                   // dims per part
  float* red_ml = reinterpret_cast<float*>(stage_mem);
  float* red_acc = red_ml + 8 * 8 * 2;
  float* cst_ml = red_acc + 8 * 8 * DW;        // [NQP][2]   (read by the cluster peers)
  float* cst_acc = cst_ml + NQP * 2;           // [NQP][D]
  {
    const int c0 = 2 * (lane & 3);
    if (lane < 4) {
      red_ml[(warp * 8 + c0) * 2 + 0] = m0;
      red_ml[(warp * 8 + c0) * 2 + 1] = l0;
      red_ml[(warp * 8 + c0 + 1) * 2 + 0] = m1;
      red_ml[(warp * 8 + c0 + 1) * 2 + 1] = l1;
    }
#pragma unroll
    for (int mt = 0; mt < KH; ++mt) {
      const int d0 = mt * 16 + (lane >> 2);
      red_acc[(warp * 8 + c0) * DW + d0] = acc[mt][0];
      red_acc[(warp * 8 + c0 + 1) * DW + d0] = acc[mt][1];
      red_acc[(warp * 8 + c0) * DW + d0 + 8] = acc[mt][2];
      red_acc[(warp * 8 + c0 + 1) * DW + d0 + 8] = acc[mt][3];
    }
  }
  __syncthreads();
  for (int e = tid; e < NQP * D; e += kSrThreads) {
    const int qr = e / D, dd = e % D;
    const int pe = dd / DW, ntq = qr >> 3, cq = qr & 7;
    float M = -INFINITY;
#pragma unroll
    for (int t = 0; t < TG; ++t) M = fmaxf(M, red_ml[((pe + DP * (ntq + NT * t)) * 8 + cq) * 2]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int t = 0; t < TG; ++t) {
      const int w = pe + DP * (ntq + NT * t);
      const float mw = red_ml[(w * 8 + cq) * 2];
      const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
      Ls += f * red_ml[(w * 8 + cq) * 2 + 1];
      A += f * red_acc[(w * 8 + cq) * DW + (dd % DW)];
    }
    cst_acc[qr * D + dd] = A;
    if (dd == 0) {
      cst_ml[qr * 2] = M;
      cst_ml[qr * 2 + 1] = Ls;
    }
  }

  // =============================================================== 4. combine over the cluster
  cluster.sync();
  float* wsm = red_ml;  // [CL][NQP] weights, then [NQP] totals (local scratch; red_* are dead)
  float* Lsm = wsm + 16 * NQP;
  if (tid < NQP) {
    float mv[kSrMaxCluster], lv[kSrMaxCluster];
#pragma unroll
    for (int q = 0; q < kSrMaxCluster; ++q) {
      mv[q] = -INFINITY;
      lv[q] = 0.f;
      if (q < CL) {
        const float* r_ml = cluster.map_shared_rank(cst_ml, q);
        mv[q] = r_ml[tid * 2];
        lv[q] = r_ml[tid * 2 + 1];
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < kSrMaxCluster; ++q) M = fmaxf(M, mv[q]);
    float Ls = 0.f;
#pragma unroll
    for (int q = 0; q < kSrMaxCluster; ++q) {
      const float f = (mv[q] == -INFINITY) ? 0.f : exp2f(mv[q] - M);
      if (q < CL) wsm[q * NQP + tid] = f;
      Ls += f * lv[q];
    }
    Lsm[tid] = Ls;
  }
  __syncthreads();
  {
    const int total = p.NQ * D;
    const int per = (total + CL - 1) / CL;
    const int e0 = rk * per, e1 = min(total, e0 + per);
    for (int e = e0 + tid; e < e1; e += kSrThreads) {
      const int qr = e / D, dd = e % D;
      float av[kSrMaxCluster];
#pragma unroll
      for (int q = 0; q < kSrMaxCluster; ++q) av[q] = (q < CL) ? cluster.map_shared_rank(cst_acc, q)[qr * D + dd] : 0.f;
      float A = 0.f;
#pragma unroll
      for (int q = 0; q < kSrMaxCluster; ++q) A += (q < CL) ? wsm[q * NQP + qr] * av[q] : 0.f;
      const int l = qr / p.G, h = g * p.G + qr % p.G;
      p.out[(((int64_t)l * p.B + b) * p.Hq + h) * D + dd] = A / Lsm[qr];
    }
  }
  cluster.sync();  // peers may read this CTA's state until every CTA is done
}

}  // namespace aoh
