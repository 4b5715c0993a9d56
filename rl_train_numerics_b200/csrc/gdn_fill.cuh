// gdn_fill.cuh -- pieces of the intra-chunk pass that the forward fill and
// the backward's per-row recomputation share: the forward workspace's header
// words, the shared-memory image of one (chunk, head) item and its loader.
#pragma once

#include "gdn_common.cuh"
#include "gdn_mma.cuh"

namespace gdn {

// Workspace header words (int32).
constexpr int kHdrError = 0;     // device error word (GDN_DEVERR_* bits)
constexpr int kHdrChunks = 1;    // number of chunks of this call
constexpr int kHdrValid = 2;     // 1 when this call's chunk table is valid
constexpr int kHdrFillNext = 3;  // work counter of k_fill
constexpr int kHdrFill0Next = 4; // work counter of the fill's first chunks (k_fill128)
constexpr int kHdrFill1Chunks = 5; // entries of the fill order (k_fill128)
constexpr int kHdrFillUniform = 6; // 1 when every sequence has the same chunk count

constexpr int kFillThreads = 128;

template <int D, class IN>
struct FillSmem {
  float k[kChunk + 1][D];  // row kChunk stays zero: the "next key" of the last token
  IN q[kChunk][D];
  IN v[kChunk][D];
  float a[kChunk];  // exp(g)
  float b[kChunk];  // beta
};

template <int RT>
__device__ __forceinline__ float pick(const float (&x)[RT], int l) {
  float val = x[0];
#pragma unroll
  for (int i = 1; i < RT; i++)
    if (l == i) val = x[i];
  return val;
}

struct FillItem {
  int c, h, n, ci, len;
  int64_t t0, L;
};

__device__ __forceinline__ FillItem fill_item(int item, int H, const int32_t* cu,
                                              const int32_t* chunk_off,
                                              const int32_t* chunk_seq) {
  FillItem it;
  it.c = item / H;
  it.h = item - it.c * H;
  it.n = chunk_seq[it.c];
  it.ci = it.c - chunk_off[it.n];
  it.L = (int64_t)cu[it.n + 1] - cu[it.n];
  it.t0 = (int64_t)cu[it.n] + (int64_t)it.ci * kChunk;
  it.len = (int)min((int64_t)kChunk, it.L - (int64_t)it.ci * kChunk);
  return it;
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Load one item's inputs into shared memory (rows past its length are zero).
template <int D, class IN>
__device__ __forceinline__ void fill_load(FillSmem<D, IN>& sm, const FillItem& it, const IN* q,
                                          const IN* k, const IN* v, const float* beta,
                                          const float* g, int H) {
  constexpr int G4 = D / 4;                        // float4 groups of a key row
  constexpr int P = (int)(D * sizeof(IN) / 16);    // 16-byte pieces of a q/v row
  constexpr int E = (int)(16 / sizeof(IN));
  const size_t tb = (size_t)it.t0 * H + it.h;
  for (int e = threadIdx.x; e < (kChunk + 1) * G4; e += kFillThreads) {
    const int r = e / G4, c = (e % G4) * 4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < it.len) x = ld4(k + (tb + (size_t)r * H) * D + c);
    *reinterpret_cast<float4*>(&sm.k[r][c]) = x;
  }
  for (int e = threadIdx.x; e < 2 * kChunk * P; e += kFillThreads) {
    const int rr = e / P, pc = (e % P) * E, r = rr % kChunk;
    IN* dst = rr < kChunk ? &sm.q[r][pc] : &sm.v[r][pc];
    const IN* src = (rr < kChunk ? q : v) + (tb + (size_t)r * H) * D + pc;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (r < it.len) x = *reinterpret_cast<const uint4*>(src);
    *reinterpret_cast<uint4*>(dst) = x;
  }
  for (int i = threadIdx.x; i < kChunk; i += kFillThreads) {
    float a = 0.f, b = 0.f;
    if (i < it.len) {
      a = step_decay(g[tb + (size_t)i * H]);
      b = beta[tb + (size_t)i * H];
    }
    sm.a[i] = a;
    sm.b[i] = b;
  }
}

// Ask L2 for an item's boundary state and input rows.
template <int D, class IN>
__device__ __forceinline__ void fill_prefetch(const FillItem& it, const float* bstate,
                                              const IN* q, const IN* k, const IN* v, int H) {
  const int tid = threadIdx.x;
  const size_t tb = (size_t)it.t0 * H + it.h;
  if (tid == 0)
    prefetch_l2(bstate + ((size_t)it.c * H + it.h) * D * D, (uint32_t)(D * D * sizeof(float)));
  if (tid < 3 * kChunk) {
    const int r = tid % kChunk;
    const IN* src = (tid < kChunk ? k : tid < 2 * kChunk ? q : v) + (tb + (size_t)r * H) * D;
    if (r < it.len) prefetch_l2(src, (uint32_t)(D * sizeof(IN)));
  }
}

// ----------------------------------------------------------------------------
// The forward fill at d = 128 (4 state rows per thread): quad reductions
// without shuffling unused values.
//
// Slot i of lane l (of its quad) holds state row r0 + (i ^ sigma(l)) with
// sigma = (0, 2, 1, 3).  The row's lane partial sum is in the same slot on
// every lane, and a reduce-scatter over the quad then needs no selects:
//   step 1 (xor 1): slot 0 += partner's slot 2, slot 1 += partner's slot 3;
//   step 2 (xor 2): slot 0 += partner's (new) slot 1.
// Lane l ends with the full sum of row r0 + sigma(l) in slot 0, equal in bits
// to the butterfly (x0 + x1) + (x2 + x3) of quad_sum: each addition adds the
// same two values (IEEE addition is commutative).  A value of the owned row
// reaches every lane's slot i from lane l ^ sigma(i) (all-gather).
// ----------------------------------------------------------------------------
__device__ __forceinline__ int quad_sigma(int l) { return ((l & 1) << 1) | (l >> 1); }

__device__ __forceinline__ float quad_rs(const float (&x)[4]) {
  const float a = __fadd_rn(x[0], __shfl_xor_sync(kFull, x[2], 1));
  const float b = __fadd_rn(x[1], __shfl_xor_sync(kFull, x[3], 1));
  return __fadd_rn(a, __shfl_xor_sync(kFull, b, 2));
}

__device__ __forceinline__ void quad_ag(float own, float (&w)[4]) {
  w[0] = own;
  w[1] = __shfl_xor_sync(kFull, own, 2);
  w[2] = __shfl_xor_sync(kFull, own, 1);
  w[3] = __shfl_xor_sync(kFull, own, 3);
}

// State slice with permuted slots: slot i <- row r0 + (i ^ sg), from the
// permuted boundary-state layout.
template <int M4>
__device__ __forceinline__ void slice4_load_bst(Slice<4, M4>& S, const float* rows, int ld,
                                                int r0, int sg, int l) {
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      const int r = r0 + (i ^ sg);
      const float4 x = ld4(rows + (size_t)r * ld + bst_col(r, group_col(l, m)));
      S.s[i][m][0] = f2(x.x, x.y);
      S.s[i][m][1] = f2(x.z, x.w);
    }
}

// The same from a row-major D x D state (h0), or zeros when rows is null.
template <int M4>
__device__ __forceinline__ void slice4_load_plain(Slice<4, M4>& S, const float* rows, int ld,
                                                  int r0, int sg, int l) {
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      const float4 x = rows ? ld4(rows + (size_t)(r0 + (i ^ sg)) * ld + group_col(l, m))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      S.s[i][m][0] = f2(x.x, x.y);
      S.s[i][m][1] = f2(x.z, x.w);
    }
}

template <int M4>
__device__ __forceinline__ void slice4_store(const Slice<4, M4>& S, float* rows, int ld, int r0,
                                             int sg, int l) {
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int m = 0; m < M4; m++)
      *reinterpret_cast<float4*>(rows + (size_t)(r0 + (i ^ sg)) * ld + group_col(l, m)) =
          make_float4(S.s[i][m][0].x, S.s[i][m][0].y, S.s[i][m][1].x, S.s[i][m][1].y);
}

template <int M4>
__device__ __forceinline__ void slice4_store_scaled(const Slice<4, M4>& S, float c, float* rows,
                                                    int ld, int r0, int sg, int l) {
  const float2 cc = f2(c, c);
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int m = 0; m < M4; m++) {
      const float2 a = __fmul2_rn(cc, S.s[i][m][0]), b = __fmul2_rn(cc, S.s[i][m][1]);
      *reinterpret_cast<float4*>(rows + (size_t)(r0 + (i ^ sg)) * ld + group_col(l, m)) =
          make_float4(a.x, a.y, b.x, b.y);
    }
}

// Shared memory of one item of the d = 128 fill: keys widened to fp32 (read
// twice per token), queries and values as bf16, and per token the step's
// scalars, computed once per item:
//   t0 = (a = exp(g), beta, c before the token, c after it),
//   t1 = (c' = a c, 1 / c' (0 when renormalising), renormalise flag, 0).
// q and v are filled by tensor-map copies (v first holds the raw keys, which
// are widened into k), counted on bar[0] (keys, queries) and bar[1] (values).
struct Fill128Smem {
  float k[kChunk + 1][128];  // row kChunk stays zero: the "next key" of the last token
  __nv_bfloat16 q[kChunk][128];
  __nv_bfloat16 v[kChunk][128];
  float4 t0[kChunk];
  float4 t1[kChunk];
  uint64_t bar[2];
};

}  // namespace gdn
