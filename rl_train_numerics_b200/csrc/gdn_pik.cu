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
// On one GPU the work is cut the same way.  A work unit is one 128 x 256 tile
// of C and one emulated rank's L / R consecutive leaves.  k_pik_gemm is
// persistent (one block per SM, units taken round-robin in a grouped raster
// that keeps a band of A rows and the B tiles beside it in L2) and
// warp-specialised:
//   warp 0      TMA producer: one 2-D box of A (128 x 64) and of B (256 x 64)
//               per 64-wide K step into a four-stage ring ("full" mbarriers
//               with transaction bytes, "empty" mbarriers from the MMAs);
//   warp 1      MMA issuer: each leaf accumulates in one of two 256-column
//               tensor-memory buffers (alternating), four m128 n256 k16 MMAs
//               per K step, ascending k, a fresh accumulator at the leaf's
//               first step; the leaf's last commit signals the epilogue;
//   warps 2-9   epilogue: read finished leaves back (one tile row and half the
//               columns per thread) and advance the balanced tree.  With two
//               or more leaves per unit they come in pairs: a pair fills both
//               buffers and is added as it is read (the tree's lowest level,
//               even leaf first), and both buffers are handed back at once.
//               The pair sums go through a binary counter: a sum is added to
//               the pending subtree sums of equal size, left operand first,
//               and the result is either the unit's sum (stored) or pushed as
//               a pending sum.  Pending sums live in a per-block slice of the
//               workspace (one 128 KB slot per level, written and read by the
//               same threads).
// The MMAs of the next leaves wait only for the pair's tensor-memory reads,
// not for the pending-sum traffic.  With R > 1 ranks the unit sums go to
// the workspace and k_pik_combine applies the levels above the ranks, again
// neighbours first.  Whatever R is, every addition of
// the tree happens in the same order on the same operands.
//
// Operands: A [M, K] and B [N, K] bf16, both K-major (row-major with K
// innermost); C [M, N] fp32.  Tiles reach shared memory by TMA in the
// 128-byte swizzled K-major layout (64 K columns = 128 bytes per row, 8-row
// atoms of 1024 bytes, 16-byte chunks permuted by the row's low three bits),
// which is also the MMA's operand layout; a k16 step starts 32 bytes further
// along the row.  Rows past M or N read as zero.  Waits are bounded: a role
// that gives up sets GDN_DEVERR_TIMEOUT in the error word and raises a shared
// abort flag so the other roles stop at their next wait; the block then waits
// (bounded) for its copies and MMAs in flight, frees tensor memory and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn_pik.h"
#include "gdn_mma.cuh"
#include "gdn_tmap.h"
#include "gdn_umma.cuh"

namespace gdn {
namespace {

constexpr int kPikBM = 128;        // tile rows (tensor-memory lanes)
constexpr int kPikBN = 256;        // tile columns (one accumulator buffer)
constexpr int kPikEpiThreads = 256;  // two warps per tensor-memory lane quarter
constexpr int kPikThreads = 64 + kPikEpiThreads;  // producer warp, MMA warp, 8 epilogue warps
constexpr int kPikChunksPerThread = kPikBN / 32 / 2;  // 32-column chunks per epilogue thread
constexpr int kPikStages = 4;
constexpr int kPikKStep = 64;      // K per stage
constexpr int kPikBand = 16;       // M tiles per band of the raster
constexpr int kPikMaxBlocks = 148; // persistent blocks at most (one per SM of a B200)
constexpr uint32_t kPikStageBytes = (kPikBM + kPikBN) * kPikKStep * 2;
constexpr int kPikPolls = 1 << 22;
constexpr int kPikErrTimeout = 4;  // GDN_DEVERR_TIMEOUT

struct PikSmem {
  __nv_bfloat16 A[kPikStages][kPikBM * kPikKStep];
  __nv_bfloat16 B[kPikStages][kPikBN * kPikKStep];
  uint64_t full[kPikStages];   // copies of the stage have landed
  uint64_t empty[kPikStages];  // MMAs reading the stage are done
  uint64_t acc_full[2];        // a leaf's MMAs into the buffer are done
  uint64_t acc_empty[2];       // the epilogue has read the buffer
  uint32_t tmem_slot;
  int abort;                   // a role gave up: the others stop
};

// 2-D tiled TMA load of one box into shared memory, completion counted on the
// mbarrier in transaction bytes.  x (the K coordinate) is a multiple of 64
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

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// Work unit u of the grouped raster: rank group z, M tile tm, N tile tn.
// Bands of kPikBand M tiles; inside a band the M tile runs fastest.
struct PikUnit {
  int z, tm, tn;
};
__device__ __forceinline__ PikUnit pik_unit(int u, int m_tiles, int n_tiles) {
  const int tiles = m_tiles * n_tiles;
  PikUnit w;
  w.z = u / tiles;
  const int t = u - w.z * tiles;
  const int per_band = kPikBand * n_tiles;
  const int band = t / per_band;
  const int r = t - band * per_band;
  const int rows = min(kPikBand, m_tiles - band * kPikBand);
  w.tm = band * kPikBand + r % rows;
  w.tn = r / rows;
  return w;
}

__device__ __forceinline__ int ctz32(uint32_t x) { return __ffs((int)x) - 1; }

// The persistent K-leaf GEMM (see the file comment).  out: C (R = 1) or the
// R rank sums [R, M, N] in the workspace; stack: kPikMaxBlocks x depth slots of
// 128 x 256 fp32 pending sums (depth = log2(L / R)).
__global__ void __launch_bounds__(kPikThreads, 1)
    k_pik_gemm(const __grid_constant__ CUtensorMap map_a,
               const __grid_constant__ CUtensorMap map_b, int M, int N, int leaf_k,
               int leaves, int n_units, float* __restrict__ out, float4* __restrict__ stack,
               int32_t* __restrict__ error) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  PikSmem& sm = *reinterpret_cast<PikSmem*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m_tiles = (M + kPikBM - 1) / kPikBM, n_tiles = (N + kPikBN - 1) / kPikBN;
  const int spl = leaf_k / kPikKStep;  // K steps per leaf
  const int depth = 31 - __clz(leaves >= 2 ? leaves / 2 : 1);  // pending-sum levels

  if (warp == 1) tmem_alloc(smem_u32(&sm.tmem_slot), 2 * kPikBN);
  if (tid == 0) {
    for (int i = 0; i < kPikStages; i++) {
      mbar_init(smem_u32(&sm.full[i]), 1);
      mbar_init(smem_u32(&sm.empty[i]), 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(smem_u32(&sm.acc_full[b]), 1);
      mbar_init(smem_u32(&sm.acc_empty[b]), kPikEpiThreads);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_slot;
  volatile int* abort_flag = &sm.abort;
  bool ok = true;
  int issued = 0;     // K steps whose copies the producer issued
  int committed = 0;  // K steps whose MMAs were issued (and committed)

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const PikUnit w = pik_unit(u, m_tiles, n_tiles);
        const int kbase = w.z * leaves * leaf_k;
        for (int step = 0; step < leaves * spl; step++, s++) {
          const int st = s % kPikStages;
          if (s >= kPikStages &&
              !mbar_wait(smem_u32(&sm.empty[st]), (uint32_t)((s / kPikStages - 1) & 1),
                         kPikPolls)) {
            ok = false;
            break;
          }
          if (*abort_flag) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm.full[st]);
          mbar_expect_tx(fb, kPikStageBytes);
          const int k0 = kbase + step * kPikKStep;
          tma_load_2d(smem_u32(sm.A[st]), &map_a, k0, w.tm * kPikBM, fb);
          tma_load_2d(smem_u32(sm.B[st]), &map_b, k0, w.tn * kPikBN, fb);
          issued = s + 1;
        }
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp == 1) {
    constexpr uint32_t idesc = idesc_bf16(kPikBM, kPikBN, false, false);
    int s = 0, lc = 0;  // K step and leaf counters of this block
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      for (int leaf = 0; leaf < leaves && ok; leaf++, lc++) {
        const int b = lc & 1, use = lc >> 1;
        // (every wait's result is made warp-uniform: the MMA wrappers need
        // the whole warp)
        if (use > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.acc_empty[b]),
                                               (uint32_t)((use - 1) & 1), kPikPolls))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * kPikBN);
        for (int ks = 0; ks < spl; ks++, s++) {
          const int st = s % kPikStages;
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.full[st]),
                                                 (uint32_t)((s / kPikStages) & 1), kPikPolls) &&
                                           !*abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sm.A[st]), b0 = smem_u32(sm.B[st]);
#pragma unroll
          for (int j = 0; j < kPikKStep / 16; j++)
            umma_bf16(d, desc_kmajor_sw128(a0 + j * 32), desc_kmajor_sw128(b0 + j * 32), idesc,
                      (ks > 0 || j > 0) ? 1u : 0u);
          umma_commit(smem_u32(&sm.empty[st]));
          committed = s + 1;
        }
        if (ok) umma_commit(smem_u32(&sm.acc_full[b]));
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
  } else {
    // Epilogue: tile row r (tensor-memory lane quarter warp % 4) and one half
    // of the tile's columns per thread (two warps per lane quarter).  Leaves
    // are read in groups of G = min(leaves, 2): a pair of leaves occupies both
    // buffers and is added (the tree's lowest level) as it is read back, then
    // both buffers are released at once; the levels above go through the
    // pending sums.
    const int q = warp & 3, r = q * 32 + lane, half = (warp - 2) >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int G = leaves >= 2 ? 2 : 1, groups = leaves / G;
    float4* my_stack = stack + (size_t)blockIdx.x * depth * (kPikBM * kPikBN / 4);
    int lc = 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const PikUnit w = pik_unit(u, m_tiles, n_tiles);
      const int m = w.tm * kPikBM + r, n0 = w.tn * kPikBN;
      float* orow = out + (size_t)w.z * M * N + (size_t)m * N + n0;
      for (int grp = 0; grp < groups; grp++) {
        bool got = true;
        for (int i = 0; i < G; i++)
          got = got && mbar_wait(smem_u32(&sm.acc_full[(lc + i) & 1]),
                                 (uint32_t)(((lc + i) >> 1) & 1), kPikPolls);
        got = __all_sync(0xffffffffu, got) && !*abort_flag;
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int b0 = lc & 1;
        float x[kPikChunksPerThread][32];
#pragma unroll
        for (int cc = 0; cc < kPikChunksPerThread; cc++) {
          const uint32_t col = (uint32_t)((half * kPikChunksPerThread + cc) * 32);
          tmem_ld32(lane_base + (uint32_t)(b0 * kPikBN) + col, x[cc]);
          if (G == 2) {
            // the odd leaf in two 16-column halves (register pressure)
#pragma unroll
            for (int hh = 0; hh < 2; hh++) {
              float y[16];
              tmem_ld16(lane_base + (uint32_t)((b0 ^ 1) * kPikBN) + col + 16 * hh, y);
              tmem_wait_ld(x[cc]);
              tmem_wait_ld(y);
#pragma unroll
              for (int e = 0; e < 16; e++)
                x[cc][16 * hh + e] = __fadd_rn(x[cc][16 * hh + e], y[e]);  // even + odd
            }
          } else {
            tmem_wait_ld(x[cc]);
          }
        }
        // every column of the group's buffers has been read: hand them back
        tc_fence_before();
        for (int i = 0; i < G; i++) mbar_arrive(smem_u32(&sm.acc_empty[(lc + i) & 1]));
        lc += G;
        // x = pending(level 0) + x, then pending(level 1) + x, ...: each
        // pending sum is the left (earlier) subtree.
        const int combos = ctz32((uint32_t)(grp + 1));
        const bool last = grp == groups - 1;
#pragma unroll 1
        for (int lev = 0; lev < combos; lev++) {
#pragma unroll
          for (int cc = 0; cc < kPikChunksPerThread; cc++) {
            const int c = half * kPikChunksPerThread + cc;
            const float4* src = my_stack + ((size_t)(lev * 8 + c) * 8) * kPikBM + r;
            // four float4 loads in flight at a time (the pair sum already
            // holds 128 registers)
#pragma unroll
            for (int f0 = 0; f0 < 8; f0 += 4) {
              float4 yv[4];
#pragma unroll
              for (int f = 0; f < 4; f++) yv[f] = src[(size_t)(f0 + f) * kPikBM];
#pragma unroll
              for (int f = 0; f < 4; f++) {
                x[cc][4 * (f0 + f) + 0] = __fadd_rn(yv[f].x, x[cc][4 * (f0 + f) + 0]);
                x[cc][4 * (f0 + f) + 1] = __fadd_rn(yv[f].y, x[cc][4 * (f0 + f) + 1]);
                x[cc][4 * (f0 + f) + 2] = __fadd_rn(yv[f].z, x[cc][4 * (f0 + f) + 2]);
                x[cc][4 * (f0 + f) + 3] = __fadd_rn(yv[f].w, x[cc][4 * (f0 + f) + 3]);
              }
              asm volatile("" ::: "memory");
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < kPikChunksPerThread; cc++) {
          const int c = half * kPikChunksPerThread + cc;
          if (last) {
            if (m < M) {
#pragma unroll
              for (int f = 0; f < 8; f++)
                if (n0 + c * 32 + 4 * f < N)
                  *reinterpret_cast<float4*>(orow + c * 32 + 4 * f) = make_float4(
                      x[cc][4 * f], x[cc][4 * f + 1], x[cc][4 * f + 2], x[cc][4 * f + 3]);
            }
          } else {
            float4* dst = my_stack + ((size_t)(combos * 8 + c) * 8) * kPikBM + r;
#pragma unroll
            for (int f = 0; f < 8; f++)
              dst[(size_t)f * kPikBM] = make_float4(x[cc][4 * f], x[cc][4 * f + 1],
                                                    x[cc][4 * f + 2], x[cc][4 * f + 3]);
          }
        }
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
  }

  const bool failed = __syncthreads_or(!ok) || *abort_flag;
  if (failed && tid == 0) {
    atomicOr(error, kPikErrTimeout);
    // Copies still in flight land before the block's shared memory is freed:
    // wait (bounded) for the last phase of every stage that was filled; then
    // for the MMAs issued (their last commit).
    for (int s = issued - kPikStages < 0 ? 0 : issued - kPikStages; s < issued; s++)
      (void)mbar_wait(smem_u32(&sm.full[s % kPikStages]), (uint32_t)((s / kPikStages) & 1),
                      kPikPolls);
  }
  if (failed && warp == 1 && committed > 0) {
    const int s = committed - 1;
    (void)mbar_wait(smem_u32(&sm.empty[s % kPikStages]), (uint32_t)((s / kPikStages) & 1),
                    kPikPolls);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 2 * kPikBN);
  if (tid == 0) {
    for (int i = 0; i < kPikStages; i++) {
      mbar_inval(smem_u32(&sm.full[i]));
      mbar_inval(smem_u32(&sm.empty[i]));
    }
    for (int b = 0; b < 2; b++) {
      mbar_inval(smem_u32(&sm.acc_full[b]));
      mbar_inval(smem_u32(&sm.acc_empty[b]));
    }
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
  int leaves;       // leaves per work unit (one rank's subtree)
  int units;        // work units: ranks x tiles
  int blocks;       // persistent blocks
  int depth;        // tree levels inside a unit = log2(leaves)
  size_t ws_ranks;  // rank sums [R, M, N] fp32 when R > 1
  size_t ws_stack;  // pending subtree sums: blocks x depth x 128 x 256 fp32
};

// Every unit is one rank's L / R leaves of one 128 x 256 tile; the grouping
// never changes the bits.
PikPlan pik_plan(int64_t M, int64_t N, int L, int R) {
  PikPlan p{};
  p.leaves = L / R;
  const int64_t tiles = ((M + kPikBM - 1) / kPikBM) * ((N + kPikBN - 1) / kPikBN);
  p.units = (int)(tiles * R);
  p.blocks = p.units < kPikMaxBlocks ? p.units : kPikMaxBlocks;
  p.depth = 0;  // levels of pending sums: the tree over the unit's leaf pairs
  while ((2 << p.depth) < p.leaves) p.depth++;
  p.ws_ranks = R > 1 ? (size_t)R * (size_t)M * (size_t)N * sizeof(float) : 0;
  p.ws_stack = (size_t)p.blocks * p.depth * kPikBM * kPikBN * sizeof(float);
  return p;
}

bool pow2(int64_t x) { return x >= 1 && (x & (x - 1)) == 0; }

int validate(int64_t M, int64_t N, int64_t K, int L, int R) {
  if (M < 0 || N < 0 || K < 0 || L < 1 || R < 1) return GDN_ERR_INVALID_ARG;
  if (!pow2(L) || !pow2(R) || L % R != 0 || L > 64) return GDN_ERR_UNSUPPORTED;
  if (N % 16 != 0 || K % ((int64_t)kPikKStep * L) != 0) return GDN_ERR_UNSUPPORTED;
  // TMA coordinates and the unit count are 32-bit.
  if (M >= 0x7fffffff || N >= 0x7fffffff || K >= 0x7fffffff) return GDN_ERR_UNSUPPORTED;
  if (((M + kPikBM - 1) / kPikBM) * ((N + kPikBN - 1) / kPikBN) * R >= 0x7fffffff)
    return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
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

int launch_gemm(const PikPlan& p, const void* A, const void* B, int64_t M, int64_t N, int64_t K,
                int64_t leaf_k, float* out, float* stack, int32_t* error, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, kPikBM) || !make_map(&mb, B, N, K, kPikBN)) return GDN_ERR_CUDA;
  // 1 KB more than the tiles need, for the 1024-byte alignment of the swizzled
  // tiles; about 194 KB keeps one block per SM, which owns all 512
  // tensor-memory columns.
  const size_t smem = sizeof(PikSmem) + 1024;
  if (cudaFuncSetAttribute(k_pik_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return GDN_ERR_CUDA;
  k_pik_gemm<<<p.blocks, kPikThreads, smem, st>>>(ma, mb, (int)M, (int)N, (int)leaf_k, p.leaves,
                                                 p.units, out, reinterpret_cast<float4*>(stack),
                                                 error);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace
}  // namespace gdn

extern "C" {

size_t gdn_pik_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_leaves, int n_ranks) {
  if (gdn::validate(M, N, K, n_leaves, n_ranks) != GDN_OK) return 0;
  if (M == 0 || N == 0 || K == 0) return 0;
  const gdn::PikPlan p = gdn::pik_plan(M, N, n_leaves, n_ranks);
  return p.ws_ranks + p.ws_stack;
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
  const size_t need = p.ws_ranks + p.ws_stack;
  if (need > 0 && (!workspace || workspace_bytes < need || !al16(workspace)))
    return GDN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  float* out = p.ws_ranks > 0 ? reinterpret_cast<float*>(ws) : C;
  float* stack = p.ws_stack > 0 ? reinterpret_cast<float*>(ws + p.ws_ranks) : nullptr;
  const int64_t leaf_k = K / n_leaves;
  int r = gdn::launch_gemm(p, A, B, M, N, K, leaf_k, out, stack, error_word, st);
  if (r != GDN_OK) return r;
  if (n_ranks > 1) {
    const int64_t MN = M * N, threads = 256, items = MN / 4;
    gdn::k_pik_combine<<<(unsigned)((items + threads - 1) / threads), (unsigned)threads, 0, st>>>(
        reinterpret_cast<const float*>(ws), n_ranks, MN, C);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  }
  return GDN_OK;
}

}  // extern "C"
