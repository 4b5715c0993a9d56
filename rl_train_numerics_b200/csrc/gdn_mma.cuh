// gdn_mma.cuh -- warp-level tensor-core helpers (mma.sync m16n8k16, bf16 in,
// fp32 accumulate), ldmatrix, cp.async, and the exact bf16 splitting of fp32
// values used by the boundary contractions.
//
// Fragment layouts (m16n8k16, g = lane / 4, t = lane % 4):
//   A (16x16, row-major): a0 = (g, 2t..2t+1), a1 = (g+8, 2t..), a2 = (g, 2t+8..),
//                         a3 = (g+8, 2t+8..)
//   B (16x8, "col")     : b0 = (k 2t..2t+1, n g), b1 = (k 2t+8.., n g)
//   C/D (16x8 fp32)     : c0,c1 = (g, 2t..2t+1), c2,c3 = (g+8, 2t..2t+1)
// so the accumulators of two adjacent n8 tiles are exactly the A fragment of
// one k16 step: the state and the walk's intermediate product stay in
// registers from one contraction to the next.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace gdn {

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// 16-byte asynchronous global -> shared copy (no mbarrier, no spin: completion
// is awaited with cp.async.wait_group, which only waits for this thread's own
// copies).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
// Programmatic dependent launch.  pdl_wait: a kernel launched as the
// dependent of the previous kernel on its stream waits here until that grid
// has completed and its writes are visible (a no-op for an ordinary launch);
// every dependent kernel calls it before it touches global memory.
// pdl_trigger: lets the dependent grid be scheduled once every block of this
// grid has passed here (it still waits for this grid's completion).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// Launches kern as the programmatic dependent of the previous kernel on st:
// its blocks may be scheduled while that kernel's last blocks run, and they
// wait (pdl_wait, first thing) until it has completed.
template <class... KArgs, class... Args>
static cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Asynchronous prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes));
}

// Exact split of an fp32 value into bf16 terms: term 0 is the round-to-nearest
// bf16 of x, every further term the round-to-nearest of what is left.  The
// residual x - hi is exact in fp32, so hi + mid + lo carries the full 24-bit
// significand (two terms carry 16 bits).
template <int NT>
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16 (&t)[NT]) {
  float r = x;
#pragma unroll
  for (int i = 0; i < NT; i++) {
    t[i] = __float2bfloat16_rn(r);
    if (i + 1 < NT) r = __fsub_rn(r, __bfloat162float(t[i]));
  }
}

__device__ __forceinline__ uint32_t pack_bf16(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// A fragments (NT split terms) of one k16 step from two adjacent accumulator
// tiles c0 (columns 0..7 of the step) and c1 (columns 8..15).
template <int NT>
__device__ __forceinline__ void acc_to_afrag(const float (&c0)[4], const float (&c1)[4],
                                             uint32_t (&a)[NT][4]) {
  __nv_bfloat16 s[4][NT], u[4][NT];
#pragma unroll
  for (int e = 0; e < 4; e++) {
    split_bf16<NT>(c0[e], s[e]);
    split_bf16<NT>(c1[e], u[e]);
  }
#pragma unroll
  for (int i = 0; i < NT; i++) {
    a[i][0] = pack_bf16(s[0][i], s[1][i]);
    a[i][1] = pack_bf16(s[2][i], s[3][i]);
    a[i][2] = pack_bf16(u[0][i], u[1][i]);
    a[i][3] = pack_bf16(u[2][i], u[3][i]);
  }
}

// Which (a-term, b-term) products a split contraction keeps: every pair whose
// combined order is below max(NA, NB), i.e. all terms down to the precision of
// the finer split.  Pairs are taken in ascending (ia + ib), then ascending ia:
// the order is part of the pinned rounding schedule.
template <int NA, int NB>
struct SplitPairs {
  static constexpr int kMax = NA > NB ? NA : NB;
  static constexpr int count() {
    int n = 0;
    for (int s = 0; s < kMax; s++)
      for (int ia = 0; ia < NA; ia++)
        if (s - ia >= 0 && s - ia < NB) n++;
    return n;
  }
  static constexpr int kCount = count();
  static constexpr int a(int p) {
    int n = 0;
    for (int s = 0; s < kMax; s++)
      for (int ia = 0; ia < NA; ia++)
        if (s - ia >= 0 && s - ia < NB) {
          if (n == p) return ia;
          n++;
        }
    return 0;
  }
  static constexpr int b(int p) {
    int n = 0;
    for (int s = 0; s < kMax; s++)
      for (int ia = 0; ia < NA; ia++)
        if (s - ia >= 0 && s - ia < NB) {
          if (n == p) return s - ia;
          n++;
        }
    return 0;
  }
};

}  // namespace gdn
