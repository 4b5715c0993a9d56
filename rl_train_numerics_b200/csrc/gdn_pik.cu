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
// above them, again neighbours first.  The group size is min(L / R, 2) for R
// emulated ranks, and whatever it is, every addition of the tree happens in
// the same order on the same operands: the result is the same for every R.
//
// Operands: A [M, K] and B [N, K] bf16, both K-major (row-major with K
// innermost); C [M, N] fp32.  Tiles reach shared memory by TMA in the
// 128-byte swizzled K-major layout: one 2-D tensor copy per operand and stage
// (64 K columns = 128 bytes per row, 8-row atoms of 1024 bytes, 16-byte
// chunks permuted by the row's low three bits), which is also the MMA's
// operand layout; a k16 step starts 32 bytes further along the row.  Rows
// past M or N read as zero.  Roles: thread 0 issues the copies
// of a stage once the MMAs that read it last have committed ("empty"
// mbarrier), warp 1 issues a stage's four MMAs once its copies have landed
// ("full" mbarrier, transaction bytes), and all four warps run the epilogue.
// Four stages.  Waits are bounded: one that gives up sets GDN_DEVERR_TIMEOUT
// in the error word, waits (bounded) for the copies and MMAs in flight, frees
// tensor memory and returns.
#include <cuda.h>
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
  uint64_t full[kPikStages];   // copies of the stage have landed
  uint64_t empty[kPikStages];  // MMAs reading the stage are done
  uint64_t done;               // every MMA is done
  uint32_t tmem_slot;
};

// 2-D tiled TMA load of one box into shared memory, completion counted on the
// mbarrier in transaction bytes.  x (the K coordinate) is a multiple of 8
// elements, so x * 2 bytes is a multiple of 16.
__device__ __forceinline__ void tma_load_2d(uint32_t sdst, const CUtensorMap* map, int x, int y,
                                            uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(sdst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}

// Descriptor of a K-major operand in the 128-byte swizzled layout: 8-row
// atoms 1024 bytes apart; the leading offset is unused within one 128-byte
// row (encoded as 16 bytes); layout type 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  return smem_desc(saddr, 16, 1024) | ((uint64_t)2 << 61);
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
    k_pik_gemm(const __grid_constant__ CUtensorMap map_a,
               const __grid_constant__ CUtensorMap map_b, int64_t M, int64_t N,
               int64_t leaf_k, float* __restrict__ out, int32_t* __restrict__ error) {
  constexpr int kCols = (G * BN < 32) ? 32 : G * BN;  // a power of two here
  constexpr uint32_t kStageBytes = (128 + BN) * kPikKStep * 2;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The swizzled tiles need 1024-byte alignment: round the base up (the
  // launch requests 1 KB more than the tiles need).
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  PikSmem<BN>& sm = *reinterpret_cast<PikSmem<BN>*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = (int)blockIdx.x * 128, n0 = (int)blockIdx.y * BN;
  const int64_t kbase = (int64_t)blockIdx.z * G * leaf_k;
  const int spl = (int)(leaf_k / kPikKStep);  // K steps per leaf
  const int S = G * spl;
  out += (int64_t)blockIdx.z * M * N;

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_slot), kCols);
  if (tid == 0) {
    for (int i = 0; i < kPikStages; i++) {
      mbar_init(smem_u32(&sm.full[i]), 1);
      mbar_init(smem_u32(&sm.empty[i]), 1);
    }
    mbar_init(smem_u32(&sm.done), 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  constexpr uint32_t idesc = idesc_bf16(128, BN, false, false);
  bool ok = true;
  int issued = 0;  // steps whose copies thread 0 issued

  if (tid == 0) {
    // Producer: the copies of step s go to stage s % NS once the MMAs of step
    // s - NS (the stage's previous use) have committed.
    for (int s = 0; s < S; s++) {
      const int st = s % kPikStages;
      if (s >= kPikStages &&
          !mbar_wait(smem_u32(&sm.empty[st]), (uint32_t)((s / kPikStages - 1) & 1), kPikPolls)) {
        ok = false;
        break;
      }
      const uint32_t fb = smem_u32(&sm.full[st]);
      mbar_expect_tx(fb, kStageBytes);
      const int k0 = (int)(kbase + (int64_t)s * kPikKStep);
      const uint32_t a0 = smem_u32(sm.A[st]), b0 = smem_u32(sm.B[st]);
      tma_load_2d(a0, &map_a, k0, m0, fb);
      tma_load_2d(b0, &map_b, k0, n0, fb);
      issued = s + 1;
    }
  } else if (warp == 1) {
    // MMA issuer: a stage's four k16 MMAs once its copies have landed.
    for (int s = 0; s < S; s++) {
      const int st = s % kPikStages;
      if (!mbar_wait(smem_u32(&sm.full[st]), (uint32_t)((s / kPikStages) & 1), kPikPolls)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(sm.A[st]), b0 = smem_u32(sm.B[st]);
      const uint32_t d = tmem + (uint32_t)((s / spl) * BN);
#pragma unroll
      for (int j = 0; j < kPikKStep / 16; j++)
        umma_bf16(d, desc_kmajor_sw128(a0 + j * 32), desc_kmajor_sw128(b0 + j * 32), idesc,
                  (s % spl != 0 || j > 0) ? 1u : 0u);
      umma_commit(smem_u32(&sm.empty[st]));
    }
    umma_commit(smem_u32(&sm.done));  // every MMA issued so far
  }
  // Everyone: wait until every MMA is done (bounded).
  if (!mbar_wait(smem_u32(&sm.done), 0u, kPikPolls)) {
    ok = false;
    (void)mbar_wait(smem_u32(&sm.done), 0u, kPikPolls);  // bounded drain before freeing
  }
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
    // Copies still in flight land before the block's shared memory is freed:
    // wait (bounded) for the last phase of every stage that was filled.
    for (int s = issued - kPikStages < 0 ? 0 : issued - kPikStages; s < issued; s++)
      (void)mbar_wait(smem_u32(&sm.full[s % kPikStages]), (uint32_t)((s / kPikStages) & 1),
                      kPikPolls);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kCols);
  if (tid == 0) {
    for (int i = 0; i < kPikStages; i++) {
      mbar_inval(smem_u32(&sm.full[i]));
      mbar_inval(smem_u32(&sm.empty[i]));
    }
    mbar_inval(smem_u32(&sm.done));
  }
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

// Group size: at most two leaves per block, so that every block runs the
// widest tile (BN = 256) and the deeper levels go to k_pik_combine.  Deeper
// in-memory trees (four or eight leaves, BN = 128 or 64) ran up to 3x slower at
// the 8192^3 shape; the grouping never changes the bits.
PikPlan pik_plan(int64_t M, int64_t N, int L, int R) {
  PikPlan p{};
  const int per_rank = L / R;  // leaves per emulated rank
  p.G = per_rank < 2 ? per_rank : 2;
  p.BN = 256;
  p.groups = L / p.G;
  p.ws = p.groups > 1 ? (size_t)p.groups * (size_t)M * (size_t)N * sizeof(float) : 0;
  return p;
}

bool pow2(int64_t x) { return x >= 1 && (x & (x - 1)) == 0; }

int validate(int64_t M, int64_t N, int64_t K, int L, int R) {
  if (M < 0 || N < 0 || K < 0 || L < 1 || R < 1) return GDN_ERR_INVALID_ARG;
  if (!pow2(L) || !pow2(R) || L % R != 0 || L > 64) return GDN_ERR_UNSUPPORTED;
  if (N % 16 != 0 || K % ((int64_t)kPikKStep * L) != 0) return GDN_ERR_UNSUPPORTED;
  // TMA coordinates are 32-bit: rows and K below 2^31.
  if (N / 64 > 65535 || M >= 0x7fffffff || N >= 0x7fffffff || K >= 0x7fffffff)
    return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Map over a [rows, K] bf16 row-major matrix with a box of 64 K columns
// (128 bytes) x box_rows rows, written to shared memory 128-byte swizzled.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kPikKStep, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Each block allocates all 512 tensor-memory columns of its SM (or 256 with
// G = 1, whose 192 KB of shared memory already keeps blocks one per SM), so
// the shared-memory request is raised to at least 116 KB: a second block on
// the SM would otherwise sit in tcgen05.alloc until the first one frees.
constexpr size_t kPikMinSmem = 116 * 1024;

template <int G, int BN>
int launch_gemm(const PikPlan& p, const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                int64_t leaf_k, float* out, int32_t* error, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, 128) || !make_map(&mb, B, N, K, BN)) return GDN_ERR_CUDA;
  auto kern = k_pik_gemm<G, BN>;
  const size_t need = sizeof(PikSmem<BN>) + 1024;
  const size_t smem = need < kPikMinSmem ? kPikMinSmem : need;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  const dim3 grid((unsigned)((M + 127) / 128), (unsigned)((N + BN - 1) / BN),
                  (unsigned)p.groups);
  kern<<<grid, kPikThreads, smem, st>>>(ma, mb, M, N, leaf_k, out, error);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
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
  float* out = p.groups > 1 ? static_cast<float*>(workspace) : C;
  const int64_t leaf_k = K / n_leaves;
  int r;
  if (p.G == 1)
    r = gdn::launch_gemm<1, 256>(p, A, B, M, N, K, leaf_k, out, error_word, st);
  else
    r = gdn::launch_gemm<2, 256>(p, A, B, M, N, K, leaf_k, out, error_word, st);
  if (r != GDN_OK) return r;
  if (p.groups > 1) {
    const int64_t MN = M * N, threads = 256, items = MN / 4;
    gdn::k_pik_combine<<<(unsigned)((items + threads - 1) / threads), (unsigned)threads, 0, st>>>(
        static_cast<const float*>(workspace), p.groups, MN, C);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  }
  return GDN_OK;
}

}  // extern "C"
