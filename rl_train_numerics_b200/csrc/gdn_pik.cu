// gdn_pik.cu -- parallelism-invariant K-leaf GEMM on the fifth-generation
// tensor core (sm_100a).
//
// "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
// section "Making kernels parallelism-invariant" (and its reduction-tree
// figure): C = A B^T with K cut into L contiguous leaves; every leaf is a
// tensor-core product with fp32 accumulation in one fixed instruction order;
// the leaves are combined by one fixed balanced binary tree; and a rank always
// owns the same contiguous block of leaves (a complete subtree), so the bits
// do not depend on how many ranks share the work.
//
// On one GPU the work is cut the same way.  k_pik_gemm<G, BN> computes, for a
// 128 x BN tile of C, one group of G consecutive leaves: each leaf
// accumulates in its own G-th of the tile's tensor-memory columns
// (G x BN <= 512), in 64-wide K steps of four m128 x BN x k16 MMAs, ascending
// k; the epilogue reads the G accumulators back and adds them level by level
// (neighbours 2i, 2i + 1).  A group is a node of the tree, so when L / G > 1
// the group sums go to a workspace and k_pik_combine applies the levels
// above them, again neighbours first.  The group size is min(L / R, 8) for R
// emulated ranks, and whatever it is, every addition of the tree happens in
// the same order on the same operands: the result is the same for every R.
//
// Operands: A [M, K] and B [N, K] bf16, both K-major (row-major with K
// innermost); C [M, N] fp32.  Tiles are staged through shared memory in the
// no-swizzle core-matrix layout by cp.async (rows past M or N are zero),
// four stages deep; an mbarrier per stage tells when the MMAs reading it are
// done.  Waits are bounded: one that gives up sets GDN_DEVERR_TIMEOUT in the
// error word, waits (bounded) for the MMAs in flight, frees tensor memory and
// returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn_pik.h"
#include "gdn_mma.cuh"
#include "gdn_umma.cuh"

namespace gdn {
namespace {

constexpr int kPikThreads = 128;   // four warps: tensor-memory lanes 0..127 = tile rows
constexpr int kPikStages = 4;
constexpr int kPikKStep = 64;      // K per stage
constexpr int kPikPolls = 1 << 22;
constexpr int kPikErrTimeout = 4;  // GDN_DEVERR_TIMEOUT

template <int BN>
struct PikSmem {
  __nv_bfloat16 A[kPikStages][128 * kPikKStep];
  __nv_bfloat16 B[kPikStages][BN * kPikKStep];
  uint64_t mbar[kPikStages];
  uint32_t tmem_slot;
};

__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
               "l"(gmem), "r"(valid ? 16 : 0));
}

// Stage the K step starting at k0: A rows m0 .. m0+127 and B rows n0 ..
// n0+BN-1, 64 columns each, into the core-matrix layout.  Eight consecutive
// threads read one row's 128 contiguous bytes.
template <int BN>
__device__ __forceinline__ void pik_stage(PikSmem<BN>& sm, int st, const __nv_bfloat16* A,
                                          const __nv_bfloat16* B, int64_t M, int64_t N,
                                          int64_t K, int64_t m0, int64_t n0, int64_t k0) {
  for (int e = threadIdx.x; e < 128 * 8; e += kPikThreads) {
    const int r = e >> 3, kg = e & 7;
    const bool ok = m0 + r < M;
    const __nv_bfloat16* src = ok ? A + (m0 + r) * K + k0 + kg * 8 : A;
    cp_async16_zfill(&sm.A[st][core_off<128>(r, kg * 8)], src, ok);
  }
  for (int e = threadIdx.x; e < BN * 8; e += kPikThreads) {
    const int r = e >> 3, kg = e & 7;
    const bool ok = n0 + r < N;
    const __nv_bfloat16* src = ok ? B + (n0 + r) * K + k0 + kg * 8 : B;
    cp_async16_zfill(&sm.B[st][core_off<BN>(r, kg * 8)], src, ok);
  }
}

template <int G>
__device__ __forceinline__ void tree16(float (&x)[G][16]) {
#pragma unroll
  for (int w = G; w > 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w / 2; i++)
#pragma unroll
      for (int j = 0; j < 16; j++) x[i][j] = __fadd_rn(x[2 * i][j], x[2 * i + 1][j]);
}

// One 128 x BN tile of one group of G leaves.  blockIdx = (M tile, N tile,
// group); out is C (one group) or the group's slice of the workspace.
template <int G, int BN>
__global__ void __launch_bounds__(kPikThreads, 1)
    k_pik_gemm(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
               int64_t M, int64_t N, int64_t K, int64_t leaf_k, float* __restrict__ out,
               int32_t* __restrict__ error) {
  constexpr int kCols = (G * BN < 32) ? 32 : G * BN;  // a power of two here
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PikSmem<BN>& sm = *reinterpret_cast<PikSmem<BN>*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = (int64_t)blockIdx.x * 128, n0 = (int64_t)blockIdx.y * BN;
  const int64_t kbase = (int64_t)blockIdx.z * G * leaf_k;
  const int spl = (int)(leaf_k / kPikKStep);  // K steps per leaf
  const int S = G * spl;
  out += (int64_t)blockIdx.z * M * N;

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_slot), kCols);
  if (tid == 0) {
    for (int i = 0; i < kPikStages; i++) mbar_init(smem_u32(&sm.mbar[i]), 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  constexpr uint32_t idesc = idesc_bf16(128, BN, false, false);

  for (int p = 0; p < kPikStages - 1; p++) {
    if (p < S) pik_stage<BN>(sm, p, A, B, M, N, K, m0, n0, kbase + (int64_t)p * kPikKStep);
    cp_async_commit();
  }
  bool ok = true;
  for (int s = 0; s < S; s++) {
    const int st = s % kPikStages;
    cp_async_wait<kPikStages - 2>();  // this thread's copies of step s are in
    fence_async_smem();
    __syncthreads();                  // everyone's are, and visible to the tensor core
    if (warp == 0) {
      tc_fence_after();
      const uint32_t a0 = smem_u32(sm.A[st]), b0 = smem_u32(sm.B[st]);
      const uint32_t d = tmem + (uint32_t)((s / spl) * BN);
#pragma unroll
      for (int j = 0; j < kPikKStep / 16; j++)
        umma_bf16(d, desc_kmajor<128>(a0 + j * 2 * 128 * 16), desc_kmajor<BN>(b0 + j * 2 * BN * 16),
                  idesc, (s % spl != 0 || j > 0) ? 1u : 0u);
      umma_commit(smem_u32(&sm.mbar[st]));
    }
    const int sn = s + kPikStages - 1;  // refill the stage step s - 1 used
    if (sn < S) {
      if (s >= 1) {
        const int sp = s - 1;
        if (!mbar_wait(smem_u32(&sm.mbar[sp % kPikStages]), (uint32_t)((sp / kPikStages) & 1),
                       kPikPolls))
          ok = false;
      }
      pik_stage<BN>(sm, sn % kPikStages, A, B, M, N, K, m0, n0,
                    kbase + (int64_t)sn * kPikKStep);
    }
    cp_async_commit();
  }
  // Every MMA is done once the last step's commit has arrived.
  const int sl = S - 1;
  const uint32_t last_bar = smem_u32(&sm.mbar[sl % kPikStages]);
  const uint32_t last_par = (uint32_t)((sl / kPikStages) & 1);
  if (!mbar_wait(last_bar, last_par, kPikPolls)) {
    ok = false;
    (void)mbar_wait(last_bar, last_par, kPikPolls);  // bounded drain before freeing
  }
  cp_async_wait<0>();
  tc_fence_after();
  const bool failed = __syncthreads_or(!ok);
  if (!failed) {
    const int64_t m = m0 + warp * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    float* orow = out + m * N + n0;
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      float x[G][16];
#pragma unroll
      for (int i = 0; i < G; i++) tmem_ld16(lane_base + (uint32_t)(i * BN + c), x[i]);
#pragma unroll
      for (int i = 0; i < G; i++) tmem_wait_ld(x[i]);
      tree16<G>(x);
      if (m < M && n0 + c < N) {
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4*>(orow + c + j) =
              make_float4(x[0][j], x[0][j + 1], x[0][j + 2], x[0][j + 3]);
      }
    }
  } else if (tid == 0) {
    atomicOr(error, kPikErrTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kCols);
  if (tid == 0)
    for (int i = 0; i < kPikStages; i++) mbar_inval(smem_u32(&sm.mbar[i]));
}

// The levels above the groups: C = tree over n_groups group sums (a power of
// two), evaluated as a binary counter so that the additions are exactly the
// balanced tree's, left operand first.
__global__ void __launch_bounds__(256)
    k_pik_combine(const float* __restrict__ parts, int n_groups, int64_t MN,
                  float* __restrict__ C) {
  const int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= MN) return;
  float4 stack[8];  // subtree sums, sizes 2^0 .. 2^6 pending at most
  int size[8];
  int top = 0;
  for (int i = 0; i < n_groups; i++) {
    float4 v = *reinterpret_cast<const float4*>(parts + (int64_t)i * MN + e);
    int sz = 1;
    while (top > 0 && size[top - 1] == sz) {
      const float4 l = stack[--top];
      v = make_float4(__fadd_rn(l.x, v.x), __fadd_rn(l.y, v.y), __fadd_rn(l.z, v.z),
                      __fadd_rn(l.w, v.w));
      sz *= 2;
    }
    stack[top] = v;
    size[top] = sz;
    top++;
  }
  *reinterpret_cast<float4*>(C + e) = stack[0];
}

struct PikPlan {
  int G, BN, groups;  // leaves per block, tile width, groups per output tile
  size_t ws;          // workspace bytes (group sums when groups > 1)
};

PikPlan pik_plan(int64_t M, int64_t N, int L, int R) {
  PikPlan p{};
  const int per_rank = L / R;  // leaves per emulated rank
  p.G = per_rank < 8 ? per_rank : 8;
  p.BN = p.G <= 2 ? 256 : 512 / p.G;
  p.groups = L / p.G;
  p.ws = p.groups > 1 ? (size_t)p.groups * (size_t)M * (size_t)N * sizeof(float) : 0;
  return p;
}

bool pow2(int64_t x) { return x >= 1 && (x & (x - 1)) == 0; }

int validate(int64_t M, int64_t N, int64_t K, int L, int R) {
  if (M < 0 || N < 0 || K < 0 || L < 1 || R < 1) return GDN_ERR_INVALID_ARG;
  if (!pow2(L) || !pow2(R) || L % R != 0 || L > 64) return GDN_ERR_UNSUPPORTED;
  if (N % 16 != 0 || K % ((int64_t)kPikKStep * L) != 0) return GDN_ERR_UNSUPPORTED;
  if (N / 64 > 65535 || (M + 127) / 128 > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

// Each block allocates all 512 tensor-memory columns of its SM (or 256 with
// G = 1, whose 192 KB of shared memory already keeps blocks one per SM), so
// the shared-memory request is raised to at least 116 KB: a second block on
// the SM would otherwise sit in tcgen05.alloc until the first one frees.
constexpr size_t kPikMinSmem = 116 * 1024;

template <int G, int BN>
cudaError_t launch_gemm(const PikPlan& p, const __nv_bfloat16* A, const __nv_bfloat16* B,
                        int64_t M, int64_t N, int64_t K, int64_t leaf_k, float* out,
                        int32_t* error, cudaStream_t st) {
  auto kern = k_pik_gemm<G, BN>;
  const size_t smem = sizeof(PikSmem<BN>) < kPikMinSmem ? kPikMinSmem : sizeof(PikSmem<BN>);
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((M + 127) / 128), (unsigned)((N + BN - 1) / BN),
                  (unsigned)p.groups);
  kern<<<grid, kPikThreads, smem, st>>>(A, B, M, N, K, leaf_k, out, error);
  return cudaGetLastError();
}

}  // namespace
}  // namespace gdn

extern "C" {

size_t gdn_pik_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_leaves, int n_ranks) {
  if (gdn::validate(M, N, K, n_leaves, n_ranks) != GDN_OK) return 0;
  return gdn::pik_plan(M, N, n_leaves, n_ranks).ws;
}

int gdn_pik_gemm(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K,
                 int n_leaves, int n_ranks, void* workspace, size_t workspace_bytes,
                 int32_t* error_word, void* stream) {
  int rc = gdn::validate(M, N, K, n_leaves, n_ranks);
  if (rc != GDN_OK) return rc;
  if (M == 0 || N == 0) return GDN_OK;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!C || !error_word || !al16(C) || (reinterpret_cast<uintptr_t>(error_word) & 3u))
    return GDN_ERR_INVALID_ARG;
  if (K == 0) {  // empty sums; A and B are not read
    return cudaMemsetAsync(C, 0, (size_t)M * N * sizeof(float),
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? GDN_OK
               : GDN_ERR_CUDA;
  }
  if (!A || !B || !al16(A) || !al16(B)) return GDN_ERR_INVALID_ARG;
  const gdn::PikPlan p = gdn::pik_plan(M, N, n_leaves, n_ranks);
  if (p.ws > 0 && (!workspace || workspace_bytes < p.ws || !al16(workspace)))
    return GDN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* a = static_cast<const __nv_bfloat16*>(A);
  const auto* b = static_cast<const __nv_bfloat16*>(B);
  float* out = p.groups > 1 ? static_cast<float*>(workspace) : C;
  const int64_t leaf_k = K / n_leaves;
  cudaError_t e;
  switch (p.G) {
    case 1: e = gdn::launch_gemm<1, 256>(p, a, b, M, N, K, leaf_k, out, error_word, st); break;
    case 2: e = gdn::launch_gemm<2, 256>(p, a, b, M, N, K, leaf_k, out, error_word, st); break;
    case 4: e = gdn::launch_gemm<4, 128>(p, a, b, M, N, K, leaf_k, out, error_word, st); break;
    default: e = gdn::launch_gemm<8, 64>(p, a, b, M, N, K, leaf_k, out, error_word, st); break;
  }
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  if (p.groups > 1) {
    const int64_t MN = M * N, threads = 256, items = MN / 4;
    gdn::k_pik_combine<<<(unsigned)((items + threads - 1) / threads), (unsigned)threads, 0, st>>>(
        static_cast<const float*>(workspace), p.groups, MN, C);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  }
  return GDN_OK;
}

}  // extern "C"
