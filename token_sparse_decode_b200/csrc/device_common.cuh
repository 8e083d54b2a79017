// Device helpers shared by the decode-step kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace aoh {

constexpr int kMaxHeads = 128;  // KV heads per cache (kernel parameters carry per-head bytes)

// ------------------------------------------------------------------ error word
// One per device (module global).  Slot 0: check id (0 = none), slots 1..3: values
// of the first failing access.  Kernels record and skip; they never trap.
enum DeviceCheck : int {
  kCheckNone = 0,
  kCheckPosition = 1,    // a stored position outside [0, L_b)
  kCheckCount = 2,       // a count or per-sequence N_fac above the row capacity
  kCheckChunk = 3,       // a chunk id outside [0, d/2)
  kCheckCapacity = 4,    // a sequence length (or an appended position) past its region's capacity
};

constexpr uint8_t kNoSlot = 255;  // head_slot entry of a KV head that a cache does not store

__device__ int g_device_error[4];

__device__ __forceinline__ void record_error(int id, int a, int b, int c) {
  if (atomicCAS(&g_device_error[0], 0, id) == 0) {
    g_device_error[1] = a;
    g_device_error[2] = b;
    g_device_error[3] = c;
  }
}

// ------------------------------------------------------------------ sequences of a cache
// Sequence b owns the tokens [offsets[b], offsets[b + 1]) of the cache (its region).
// Without per-sequence lengths it fills the region; with them it holds positions
// 0 .. lengths[b] - 1.  In the linear layout position p is token offsets[b] + p, so a
// length beyond the region is recorded (check 4) and clamped to it; a ring keeps only
// some positions (see ring_slot) and its length is not bounded by the region.
__device__ __forceinline__ int seq_length(const int32_t* offsets, const int32_t* lengths, int b, bool ring,
                                          int* off_out) {
  const int off = offsets[b];
  const int cap = offsets[b + 1] - off;
  *off_out = off;
  if (!lengths) return cap;
  int L = lengths[b];
  if (L < 0 || (!ring && L > cap)) {
    record_error(kCheckCapacity, b, L, cap);
    L = L < 0 ? 0 : cap;
  }
  return L;
}

// Slot of position p in a ring of `sink` + `window` slots: positions below the sink keep
// their own slot, later ones take the window slots in turn (the caller reads only
// positions the ring still holds: [0, min(sink, L)) and [max(sink, L - window), L)).
__device__ __forceinline__ int ring_slot(int p, int sink, int window) {
  return (p < sink || window <= 0) ? p : sink + (p - sink) % window;
}

// ------------------------------------------------------------------ bf16 unpacking
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Order-preserving map of a finite fp32 to uint32 (larger float -> larger key);
// -0 is folded onto +0 so that the two compare equal.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// fp32 dot of 8 bf16 (one 16-byte segment) with 8 fp32 weights, in element order
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

// ------------------------------------------------------------------ async copies
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy; when !valid the destination is zero-filled and
// nothing is read.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// wait_group with a run-time count (the instruction takes an immediate)
__device__ __forceinline__ void cp_async_wait_n(int n) {
  switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    default: cp_async_wait<6>(); break;
  }
}

// 16 bytes of read-only data that is used once: not kept in L1
__device__ __forceinline__ uint4 ld_stream_v4(const uint16_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ------------------------------------------------------------------ tensor-core fragments
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Transpose an 8x8 b16 matrix held one 32-bit pair per lane.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// ------------------------------------------------------------------ programmatic dependent launch
// A kernel launched with programmatic stream serialization may be scheduled while the kernel
// before it on the stream is still running.  grid_dep_wait() blocks until that kernel has
// completed and its writes are visible (a no-op when the launch has no such dependency);
// every kernel launched that way calls it before it reads or writes global memory.
// grid_dep_launch() lets the next such launch begin scheduling its CTAs.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ------------------------------------------------------------------ split cluster barrier
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// ------------------------------------------------------------------ small reductions

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024, multiple of 32).
// `scratch` holds >= 33 ints of shared memory.  Returns the exclusive prefix; *total
// receives the block sum.  Must be called by every thread of the block.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
    int s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nwarps) scratch[lane] = s - w;  // exclusive warp offsets
    if (lane == 31) scratch[32] = s;
  }
  __syncthreads();
  int res = scratch[warp] + x - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}

}  // namespace aoh
