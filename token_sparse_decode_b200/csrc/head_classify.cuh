// AoH offline head classifier (AoH summary, Resumen Técnico: Autonomía de Cabezales,
// Metodología §1-§4).
//
// For q head h with key block of KV head g = h / G (W^h = rows h*d .. (h+1)*d of a
// projection weight [H*d, d_model]):
//   §1  the frozen query-key kernel M_h = W_K^T W_Q (d_model x d_model);
//   §3  its non-zero singular values are sqrt(eig(C_h)) with the d x d proxy
//       C_h = A_h B_g, A_h = W_Q^h W_Q^h^T, B_g = W_K^g W_K^g^T (Sylvester);
//   §2  ER(h) = exp(-sum sigma_hat log sigma_hat), sigma_hat = sigma / sum sigma;
//   §4  GQA: the group's ER is the mean over its q heads; the n_retrieval lowest groups
//       are retrieval heads (DENSE), the others streaming heads (STREAM).
//
// Kernels:
//   gram_kernel      A_h and B_g for every head: [d x d_model] x [d_model x d] on the fp64
//                    tensor-core path (mma.sync m8n8k4 f64): the bf16 weights are exact in
//                    fp64, so products are exact and sums round in fp64 (the fp32
//                    accumulation of the bf16 path moved ER by up to 2.6e-4 on
//                    concentrated spectra); d_model split over CTAs, fp64 partials;
//   gram_reduce      the partials summed in a fixed order in fp64 (deterministic);
//   spectrum_kernel  one CTA per q head, fp64 in shared memory: Cholesky B = L L^T, then
//                    S = L^T A L (symmetric, eig(S) = eig(A B) = eig(C_h)), its eigenvalues
//                    by cyclic Jacobi (parallel round-robin pairs, at most kJacobiSweeps
//                    sweeps, stopping when the off-diagonal sum of squares is below 1e-26
//                    of the diagonal's), then sigma = sqrt(max(lambda, 0)) and ER;
//   group_roles      group means and the ranking (equal ER: the lower KV head first).
// A B_g that is not positive definite (W_K^g without full row rank) has no Cholesky
// factor: the head's ER is written as NaN and device check 5 is recorded.
#pragma once

#include "device_common.cuh"

namespace aoh {

constexpr int kGramThreads = 256;
constexpr int kGramK = 64;            // d_model columns per pipeline stage
constexpr int kGramPitch = kGramK + 8;  // bf16 elements per smem row (144 B: ldmatrix without conflicts)
constexpr int kGramStages = 3;
constexpr int kSpecThreads = 256;
constexpr int kJacobiSweeps = 40;
constexpr int kCheckFactor = 5;       // device check id: a key Gram matrix without a Cholesky factor

struct GramParams {
  const uint16_t* wq;   // [Hq * D][d_model]
  const uint16_t* wk;   // [Hkv * D][d_model]
  double* partial;      // [Hq + Hkv][splits][D][D]
  int32_t d_model, Hq, Hkv, splits, k_per_split;
};

// D = A(8x4, row) * B(4x8, col) + C on the fp64 tensor-core path
__device__ __forceinline__ void dmma_884(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

__device__ __forceinline__ double bf16_at(const uint16_t* t, int r, int c) {
  return (double)__uint_as_float((uint32_t)t[r * kGramPitch + c] << 16);
}

// One CTA: half of the columns (blockIdx.z) of a head's W W^T over one split of d_model, on the
// fp64 tensor-core path: bf16 weights are exact in fp64, so every product is exact and the sums
// carry fp64 rounding only.  8 warps as 4 (rows) x 2 (columns) of 8 x 8 tiles.
template <int D>
__global__ void __launch_bounds__(kGramThreads) gram_kernel(const GramParams p) {
  constexpr int WM = D / 4, WN = D / 4;  // warp tile; the CTA covers D rows x D/2 columns
  constexpr int MT = WM / 8, NT = WN / 8;
  constexpr int kStageElems = D * kGramPitch;
  extern __shared__ __align__(16) uint16_t gsm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int head = blockIdx.y, split = blockIdx.x, half = blockIdx.z;
  const uint16_t* w = head < p.Hq ? p.wq + (int64_t)head * D * p.d_model
                                  : p.wk + (int64_t)(head - p.Hq) * D * p.d_model;
  const int k0 = split * p.k_per_split;
  const int nsteps = p.k_per_split / kGramK;
  const uint32_t sbase = smem_u32(gsm);

  auto issue = [&](int st) {
    if (st < nsteps) {
      const uint32_t dst = sbase + (uint32_t)((st % kGramStages) * kStageElems) * 2;
      for (int c = tid; c < D * (kGramK / 8); c += kGramThreads) {
        const int r = c / (kGramK / 8), ch = c % (kGramK / 8);
        cp_async_16(dst + (uint32_t)(r * kGramPitch + ch * 8) * 2, w + (int64_t)r * p.d_model + k0 + st * kGramK + ch * 8,
                    true);
      }
    }
    cp_async_commit();
  };

  const int wm = warp & 3, wn = warp >> 2;
  const int row0 = wm * WM, col0 = half * (D / 2) + wn * WN;
  const int gr = lane >> 2, gc = lane & 3;  // fragment row (A) / column (B), and k within the step
  double acc[MT][NT][2];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

#pragma unroll
  for (int s = 0; s < kGramStages - 1; ++s) issue(s);
  for (int st = 0; st < nsteps; ++st) {
    cp_async_wait<kGramStages - 2>();
    __syncthreads();
    issue(st + kGramStages - 1);
    const uint16_t* tile = gsm + (st % kGramStages) * kStageElems;
#pragma unroll 4
    for (int kk = 0; kk < kGramK; kk += 4) {
      double a[MT], b[NT];
#pragma unroll
      for (int i = 0; i < MT; ++i) a[i] = bf16_at(tile, row0 + i * 8 + gr, kk + gc);  // A[i][k] = W[i][k]
#pragma unroll
      for (int j = 0; j < NT; ++j) b[j] = bf16_at(tile, col0 + j * 8 + gr, kk + gc);  // B[k][j] = W[j][k]
#pragma unroll
      for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < NT; ++j) dmma_884(acc[i][j], a[i], b[j]);
    }
  }
  cp_async_wait<0>();
  double* out = p.partial + ((int64_t)head * p.splits + split) * D * D;
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int r = row0 + i * 8 + gr, c = col0 + j * 8 + 2 * gc;
      out[r * D + c] = acc[i][j][0];
      out[r * D + c + 1] = acc[i][j][1];
    }
}

// gram[h][i][j] = sum over splits s (in order) of partial[h][s][i][j], in fp64
__global__ void __launch_bounds__(256) gram_reduce_kernel(const double* partial, double* gram, int64_t n_heads,
                                                          int splits, int dd) {
  const int64_t total = n_heads * dd;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t h = e / dd, ij = e % dd;
    double s = 0.0;
    for (int t = 0; t < splits; ++t) s += partial[(h * splits + t) * dd + ij];
    gram[e] = s;
  }
}

struct SpectrumParams {
  const double* gram;   // [Hq + Hkv][D][D]: A_h for q heads, then B_g
  double* work;         // [Hq][D][D] scratch (S of each head)
  double* er_heads;     // [Hq]
  int32_t Hq, Hkv, G;
};

// Shared-memory matrix of D x D doubles with a row pitch of D + 1 (column walks without bank
// conflicts).
template <int D>
__device__ __forceinline__ double& mat(double* X, int i, int j) { return X[i * (D + 1) + j]; }

template <int D>
__device__ double block_sum(double v, double* red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < kSpecThreads / 32; ++w) t += red[w];  // fixed order: the same bits every run
  return t;
}

template <int D>
__global__ void __launch_bounds__(kSpecThreads) spectrum_kernel(const SpectrumParams p) {
  extern __shared__ __align__(16) double X[];  // [D][D + 1]
  __shared__ double s_c[D / 2], s_s[D / 2];
  __shared__ double red[kSpecThreads / 32];
  __shared__ int s_fail;
  double* TJ = X + D * (D + 1);                 // [D][8] block of T = A L
  const int tid = threadIdx.x;
  const int h = blockIdx.x, g = h / p.G;
  const double* A = p.gram + (int64_t)h * D * D;
  const double* Bg = p.gram + ((int64_t)p.Hq + g) * D * D;
  double* S = p.work + (int64_t)h * D * D;

  // ---- Cholesky of B_g in place (lower triangle), right-looking
  for (int e = tid; e < D * D; e += kSpecThreads) mat<D>(X, e / D, e % D) = Bg[e];
  if (tid == 0) s_fail = 0;
  __syncthreads();
  for (int j = 0; j < D; ++j) {
    const double piv = mat<D>(X, j, j);
    if (!(piv > 0.0)) {  // uniform: every thread reads the same pivot
      if (tid == 0) {
        s_fail = 1;
        record_error(kCheckFactor, h, j, 0);
      }
      break;
    }
    const double ljj = sqrt(piv);
    for (int i = j + 1 + tid; i < D; i += kSpecThreads) mat<D>(X, i, j) /= ljj;
    __syncthreads();
    if (tid == 0) mat<D>(X, j, j) = ljj;
    // trailing update of the lower triangle: X[i][k] -= L[i][j] L[k][j] for j < k <= i
    const int m = D - 1 - j;
    for (int e = tid; e < m * m; e += kSpecThreads) {
      const int i = j + 1 + e / m, k = j + 1 + e % m;
      if (k <= i) mat<D>(X, i, k) -= mat<D>(X, i, j) * mat<D>(X, k, j);
    }
    __syncthreads();
  }
  __syncthreads();  // s_fail, written by thread 0 when a pivot fails, is read by every thread
  if (s_fail) {
    if (tid == 0) p.er_heads[h] = __longlong_as_double(0x7ff8000000000000ll);
    return;
  }
  for (int e = tid; e < D * D; e += kSpecThreads) {  // zero the strict upper triangle: X = L
    const int i = e / D, k = e % D;
    if (k > i) mat<D>(X, i, k) = 0.0;
  }
  __syncthreads();

  // ---- S = L^T A L, eight columns at a time: T_J = A L[:, J], S[:, J] = L^T T_J
  for (int J = 0; J < D; J += 8) {
    for (int e = tid; e < D * 8; e += kSpecThreads) {
      const int i = e >> 3, jj = e & 7;
      double t = 0.0;
      for (int k = J + jj; k < D; ++k) t += A[(int64_t)i * D + k] * mat<D>(X, k, J + jj);  // L[k][J+jj] = 0 for k < J+jj
      TJ[i * 8 + jj] = t;
    }
    __syncthreads();
    for (int e = tid; e < D * 8; e += kSpecThreads) {
      const int i = e >> 3, jj = e & 7;
      double t = 0.0;
      for (int k = i; k < D; ++k) t += mat<D>(X, k, i) * TJ[k * 8 + jj];  // L^T[i][k] = L[k][i], zero for k < i
      S[(int64_t)i * D + J + jj] = t;
    }
    __syncthreads();
  }
  // S is symmetric up to rounding: use its lower triangle for both halves
  for (int e = tid; e < D * D; e += kSpecThreads) {
    const int i = e / D, k = e % D;
    mat<D>(X, i, k) = i >= k ? S[(int64_t)i * D + k] : S[(int64_t)k * D + i];
  }
  __syncthreads();

  // ---- eigenvalues of S: cyclic Jacobi, D/2 disjoint pairs per round, D - 1 rounds a sweep
  constexpr int NP = D / 2;
  for (int sweep = 0; sweep < kJacobiSweeps; ++sweep) {
    double off = 0.0, dg = 0.0;
    for (int e = tid; e < D * D; e += kSpecThreads) {
      const int i = e / D, k = e % D;
      const double x = mat<D>(X, i, k);
      if (i == k) dg += x * x; else off += x * x;
    }
    off = block_sum<D>(off, red);
    dg = block_sum<D>(dg, red);
    if (off <= 1e-26 * dg) break;  // uniform (1e-13 relative: the level fp64 rounding leaves)
    for (int round = 0; round < D - 1; ++round) {
      // round-robin pairing: player 0 stays, the others rotate
      if (tid < NP) {
        const int a = tid == 0 ? 0 : 1 + (tid - 1 + round) % (D - 1);
        const int b = 1 + (D - 1 - tid - 1 + round) % (D - 1);
        const int pp = min(a, b), qq = max(a, b);
        const double apq = mat<D>(X, pp, qq);
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (mat<D>(X, qq, qq) - mat<D>(X, pp, pp)) / (2.0 * apq);
          const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        s_c[tid] = c;
        s_s[tid] = s;
      }
      __syncthreads();
      // rows: X <- J^T X
      for (int e = tid; e < NP * D; e += kSpecThreads) {
        const int k = e / D, col = e % D;
        const int a = k == 0 ? 0 : 1 + (k - 1 + round) % (D - 1);
        const int b = 1 + (D - 1 - k - 1 + round) % (D - 1);
        const int pp = min(a, b), qq = max(a, b);
        const double c = s_c[k], s = s_s[k];
        const double x = mat<D>(X, pp, col), y = mat<D>(X, qq, col);
        mat<D>(X, pp, col) = c * x - s * y;
        mat<D>(X, qq, col) = s * x + c * y;
      }
      __syncthreads();
      // columns: X <- X J
      for (int e = tid; e < NP * D; e += kSpecThreads) {
        const int k = e / D, row = e % D;
        const int a = k == 0 ? 0 : 1 + (k - 1 + round) % (D - 1);
        const int b = 1 + (D - 1 - k - 1 + round) % (D - 1);
        const int pp = min(a, b), qq = max(a, b);
        const double c = s_c[k], s = s_s[k];
        const double x = mat<D>(X, row, pp), y = mat<D>(X, row, qq);
        mat<D>(X, row, pp) = c * x - s * y;
        mat<D>(X, row, qq) = s * x + c * y;
      }
      __syncthreads();
    }
  }

  // ---- sigma = sqrt(max(lambda, 0)); ER over the values above 1e-12 of the largest
  double sig = 0.0;
  if (tid < D) sig = sqrt(fmax(mat<D>(X, tid, tid), 0.0));
  double mx = sig;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  __syncthreads();
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = 0.0;
  for (int w = 0; w < kSpecThreads / 32; ++w) mx = fmax(mx, red[w]);
  const bool keep = tid < D && sig > 1e-12 * mx;
  const double total = block_sum<D>(keep ? sig : 0.0, red);
  double ent = 0.0;
  if (keep) {
    const double q = sig / total;
    ent = -q * log(q);
  }
  ent = block_sum<D>(ent, red);
  if (tid == 0) p.er_heads[h] = total > 0.0 ? exp(ent) : 0.0;
}

struct RolesParams {
  const double* er_heads;  // [Hq]
  double* er_groups;       // [Hkv]
  uint8_t* roles;          // [Hkv]
  int32_t Hkv, G, n_retrieval;
};

__global__ void __launch_bounds__(128) group_roles_kernel(const RolesParams p) {
  __shared__ double s_er[128];
  const int g = threadIdx.x;
  if (g < p.Hkv) {
    double s = 0.0;
    for (int i = 0; i < p.G; ++i) s += p.er_heads[g * p.G + i];
    s_er[g] = s / p.G;
    p.er_groups[g] = s_er[g];
  }
  __syncthreads();
  if (g < p.Hkv) {
    int rank = 0;  // groups ordered before g: lower ER, or equal ER and a lower index
    for (int o = 0; o < p.Hkv; ++o) rank += (s_er[o] < s_er[g]) || (s_er[o] == s_er[g] && o < g);
    p.roles[g] = rank < p.n_retrieval ? 1 : 2;  // DENSE (retrieval) : STREAM
  }
}

}  // namespace aoh
