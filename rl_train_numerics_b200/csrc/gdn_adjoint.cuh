// gdn_adjoint.cuh -- the adjoint of the CPR backward in chunk form (bf16
// inputs): a chunk-parallel prep, a serial reverse walk over chunk ends, and
// a chunk-parallel solve for the per-token vectors w.
//
// The token recurrence of the adjoint (gdn_backward.cu's header), per
// (sequence, head) and chunk of length L with T = (I + A)^{-1} of the
// forward's boundary prep, Tb = T diag(beta e^G), dvec = e^{G_{L-1} - G},
// gamma = e^{G_{L-1}} and Pm[r][t] = [t <= r] e^{G_r - G_t} q_r . k_t,
// unrolls to
//   X       = scale (diag(e^G) Q - Pm Tb K)                         (L x d_k)
//   mu_a    = gamma mu_e - ((mu_e K^T) diag(dvec)) Tb K + DO^T X     (the
//             chunk map of the adjoint: the forward boundary map's linear
//             part transposed, plus the chunk's own do terms)
//   W       = T^T (diag(dvec) (mu_e K^T)^T + scale Pm^T DO)          (L x d_v)
// with mu_e the adjoint at the chunk's end and mu_a at its start (the end of
// the chunk before).  The identities are exact (pinned in float64 by
// tests/test_backward_algebra.py); the kernels evaluate them on the tensor
// cores (mma.sync m16n8k16) with every fp32 operand split exactly into three
// bf16 terms and all term pairs down to the third term's order accumulated in
// fp32 (fp32 accuracy; keys, queries and do are exact in bf16).  The walk is
// the only serial part: a chain of L x d x d products per chunk instead of the
// token scan's chain per token.
//   k_adj_prep  per (chunk, head): the forward prep's T (trailing partial
//               chunks zero-padded), Pm, X; writes the chunk's adjoint pack
//   k_adj_walk  per (sequence, head, 64 state rows), last chunk first: mu at
//               every chunk end, dh0, and Ydv = (mu_e K^T) diag(dvec)
//   adj_w_item  per (chunk, head): W -> w and dv = beta w (launched with the
//               chunk u of the backward, gdn_backward.cu's k_bwd_wu)
#pragma once

#include <cuda.h>

#include <cstddef>

#include "gdn_boundary.cuh"
#include "gdn_fill.cuh"

namespace gdn {

constexpr int kAdjNT = 3;  // bf16 terms of an fp32 operand

// The adjoint pack of one (chunk, head).  Planes are bf16 in the core layout
// (64 rows); the walk bulk-copies the head, the keys, X and Tb, the solve the
// rest.  The do rows are not in it: both read them from the input (the walk
// by a tensor-map copy of its rows' columns, the solve by cp.async).
template <int D>
struct AdjPack {
  float dvec[kChunk];
  float beta[kChunk];  // 0 past the chunk's length
  float gamma[4];      // [0] = e^{G_{L-1}}
  __nv_bfloat16 K[1][kChunk * D];               // [t][j]
  __nv_bfloat16 X[kAdjNT][kChunk * D];          // [t][j]
  __nv_bfloat16 Tb[kAdjNT][kChunk * kChunk];    // [t][m], m <= t
  __nv_bfloat16 T[kAdjNT][kChunk * kChunk];     // [m][t], t <= m
  __nv_bfloat16 Pm[kAdjNT][kChunk * kChunk];    // [r][t], t <= r
};
template <int D>
constexpr size_t adj_pack_bytes() {
  return round_up(sizeof(AdjPack<D>), 128);
}

// Three-term split of (x0, x1) stored as bf16 pairs at element offset off of
// three planes nelem elements apart.
__device__ __forceinline__ void put3(__nv_bfloat16* p, size_t nelem, int off, float x0, float x1) {
  __nv_bfloat16 a[kAdjNT], b[kAdjNT];
  split_bf16<kAdjNT>(x0, a);
  split_bf16<kAdjNT>(x1, b);
#pragma unroll
  for (int q = 0; q < kAdjNT; q++)
    *reinterpret_cast<uint32_t*>(p + q * nelem + off) = pack_bf16(a[q], b[q]);
}

// ----------------------------------------------------------------------------
// k_adj_prep
// ----------------------------------------------------------------------------
// The queries go where the prep's fp32 T was, once T is split; the prep's head
// takes the Tb terms.
template <int D>
struct AdjPrepSmem {
  PrepSmem<D, __nv_bfloat16> prep;
  union {
    PrepAT AT;
    __nv_bfloat16 Q[1][kChunk * D];
  };
};

template <int D>
__global__ void __launch_bounds__(kBndThreads, 3)
    k_adj_prep(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
               const float* __restrict__ beta,
               const float* __restrict__ g, const int32_t* __restrict__ cu, int H, float scale,
               const int32_t* __restrict__ hdr, const int32_t* __restrict__ chunk_off,
               const int32_t* __restrict__ chunk_seq, char* __restrict__ apacks) {
  using bf16 = __nv_bfloat16;
  constexpr int C = kChunk, PL = C * C, PD = C * D;
  static_assert(sizeof(PackHead<D, bf16>) >= kAdjNT * PL * sizeof(bf16), "Tb terms fit the head");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AdjPrepSmem<D>& sm = *reinterpret_cast<AdjPrepSmem<D>*>(smem_raw);
  // Launched as a programmatic dependent of the kernel before it (the
  // forward's fill or walk), whose outputs it does not read: it starts in
  // that grid's tail and waits for it only before it ends, so that this grid,
  // and everything after it, completes after it.  The chunk table it reads
  // completed before that kernel started.
  pdl_trigger();  // the reverse walk may be scheduled; it waits for this grid
  if (hdr[kHdrValid] != 1) {
    pdl_wait();
    return;
  }
  const int c = blockIdx.x, h = blockIdx.y;
  if (c >= hdr[kHdrChunks]) {
    pdl_wait();
    return;
  }
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const FillItem it = fill_item(c * H + h, H, cu, chunk_off, chunk_seq);
  const int len = it.len;
  const size_t tok = (size_t)it.t0 * H + h;
  AdjPack<D>& pk = *reinterpret_cast<AdjPack<D>*>(apacks + ((size_t)c * H + h) * adj_pack_bytes<D>());

  prep_stage<D, bf16>(sm.prep, k + tok * D, (size_t)H * D, beta + tok, g + tok, (size_t)H, len);
  bnd_prep<D, bf16>(sm.prep, sm.AT);

  if (tid < C) {
    pk.dvec[tid] = sm.prep.head.dvec[tid];
    pk.beta[tid] = sm.prep.beta[tid];
  }
  if (tid < 4) pk.gamma[tid] = sm.prep.head.gamma[tid];
  for (int e = tid; e < PD / 8; e += kBndThreads)
    reinterpret_cast<uint4*>(pk.K[0])[e] = reinterpret_cast<const uint4*>(sm.prep.K[0])[e];
  // T (rows m, columns t) and Tb = T diag(beta e^G) (rows t, columns m).
  bf16* tb3 = reinterpret_cast<bf16*>(&sm.prep.head);
  for (int e = tid; e < PL / 2; e += kBndThreads) {
    const int i = e / (C / 2), j = 2 * (e % (C / 2));
    const float t0 = i >= j ? sm.AT[i][j] : 0.f, t1 = i >= j + 1 ? sm.AT[i][j + 1] : 0.f;
    const float b0 = __fmul_rn(t0, sm.prep.bg[j]), b1 = __fmul_rn(t1, sm.prep.bg[j + 1]);
    const int off = core_off<C>(i, j);
    put3(pk.T[0], PL, off, t0, t1);
    put3(pk.Tb[0], PL, off, b0, b1);
    put3(tb3, PL, off, b0, b1);
  }
  __syncthreads();  // T is read: its space takes the queries
  stage_planes<D, bf16>(sm.Q, q + tok * D, (size_t)H * D, kBndThreads, len);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // Pm on warp w's rows 16w .. 16w + 15 (n8 tiles up to the diagonal block).
  float pm[8][4];
#pragma unroll
  for (int n = 0; n < 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) pm[n][e] = 0.f;
#pragma unroll 2
  for (int ks = 0; ks < D / 16; ks++) {
    uint32_t a[4];
    ldsm_x4(a, afrag_addr(sm.Q[0], 16 * w, 16 * ks));
#pragma unroll
    for (int np = 0; np < 4; np++) {
      if (np <= w) {
        uint32_t b[4];
        ldsm_x4(b, bfrag_nk_addr(sm.prep.K[0], 16 * np, 16 * ks));
        mma16816(pm[2 * np], a, b[0], b[1]);
        mma16816(pm[2 * np + 1], a, b[2], b[3]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int r = 16 * w + gq + 8 * (e >> 1), t = 8 * n + 2 * tq + (e & 1);
      pm[n][e] = (t <= r && r < len)
                     ? __fmul_rn(expf(__double2float_rn(sm.prep.G[r] - sm.prep.G[t])), pm[n][e])
                     : 0.f;
    }
#pragma unroll
  for (int n = 0; n < 8; n++)
#pragma unroll
    for (int hf = 0; hf < 2; hf++)
      put3(pk.Pm[0], PL, core_off<C>(16 * w + gq + 8 * hf, 8 * n + 2 * tq), pm[n][2 * hf],
           pm[n][2 * hf + 1]);

  // Y2 = Pm Tb on the same rows (both lower triangular).
  float y2[8][4];
#pragma unroll
  for (int n = 0; n < 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) y2[n][e] = 0.f;
  using P33 = SplitPairs<kAdjNT, kAdjNT>;
  using P31 = SplitPairs<kAdjNT, 1>;
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    if (ks > w) continue;
    uint32_t a[kAdjNT][4];
    acc_to_afrag<kAdjNT>(pm[2 * ks], pm[2 * ks + 1], a);
#pragma unroll
    for (int np = 0; np < 4; np++) {
      if (np > ks) continue;
      uint32_t b[kAdjNT][4];
#pragma unroll
      for (int qq = 0; qq < kAdjNT; qq++) ldsm_x4_t(b[qq], bfrag_kn_addr(tb3 + qq * PL, 16 * ks, 16 * np));
#pragma unroll
      for (int p = 0; p < P33::kCount; p++) {
        mma16816(y2[2 * np], a[P33::a(p)], b[P33::b(p)][0], b[P33::b(p)][1]);
        mma16816(y2[2 * np + 1], a[P33::a(p)], b[P33::b(p)][2], b[P33::b(p)][3]);
      }
    }
  }
  // X = scale (e^{G_r} q_r - (Y2 K)_r), rows of this warp.
  float x[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) x[n][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    if (ks > w) continue;
    uint32_t a[kAdjNT][4];
    acc_to_afrag<kAdjNT>(y2[2 * ks], y2[2 * ks + 1], a);
#pragma unroll
    for (int np = 0; np < D / 16; np++) {
      uint32_t b[4];
      ldsm_x4_t(b, bfrag_kn_addr(sm.prep.K[0], 16 * ks, 16 * np));
#pragma unroll
      for (int p = 0; p < P31::kCount; p++) {
        mma16816(x[2 * np], a[P31::a(p)], b[0], b[1]);
        mma16816(x[2 * np + 1], a[P31::a(p)], b[2], b[3]);
      }
    }
  }
#pragma unroll
  for (int hf = 0; hf < 2; hf++) {
    const int r = 16 * w + gq + 8 * hf;
    const float eg = expf(__double2float_rn(sm.prep.G[r]));
#pragma unroll
    for (int n = 0; n < D / 8; n++) {
      const int j = 8 * n + 2 * tq, off = core_off<C>(r, j);
      const __nv_bfloat162 qv = *reinterpret_cast<const __nv_bfloat162*>(&sm.Q[0][off]);
      const float x0 = __fmul_rn(scale, __fsub_rn(__fmul_rn(eg, __low2float(qv)), x[n][2 * hf]));
      const float x1 =
          __fmul_rn(scale, __fsub_rn(__fmul_rn(eg, __high2float(qv)), x[n][2 * hf + 1]));
      put3(pk.X[0], PD, off, x0, x1);
    }
  }
  pdl_wait();  // the kernel before it (see above)
}

// ----------------------------------------------------------------------------
// k_adj_walk
// ----------------------------------------------------------------------------
// A block takes 32 state rows of one (sequence, head): two pairs of warps,
// 16 rows per pair; the pair's two warps hold columns 0 .. D/2 - 1 and
// D/2 .. D - 1 of those rows.  (64-row blocks, eight warps to an SM, made
// each chunk step slower: 0.84 against 0.64 ms on the trainer batch.)
constexpr int kAdjWalkRows = 32;
constexpr int kAdjWalkPairs = kAdjWalkRows / 16;
constexpr int kAdjWalkThreads = 64 * kAdjWalkPairs;

// One chunk's walk operands in shared memory: the pack's head and keys, the
// do columns of the block's rows (their core-layout column groups, a
// tensor-map destination), X and Tb.
template <int D>
struct AdjWalkBuf {
  float dvec[kChunk];
  float beta[kChunk];
  float gamma[4];
  __nv_bfloat16 K[1][kChunk * D];                           // [t][j]
  alignas(128) __nv_bfloat16 DOr[1][kChunk * kAdjWalkRows];  // [t][i - first row of the block]
  __nv_bfloat16 X[kAdjNT][kChunk * D];            // [t][j]
  __nv_bfloat16 Tb[kAdjNT][kChunk * kChunk];      // [t][m], m <= t
};
template <int D>
constexpr uint32_t adj_walk_head_bytes() {
  return (uint32_t)offsetof(AdjPack<D>, X);
}
template <int D>
constexpr uint32_t adj_walk_xtb_bytes() {
  return (uint32_t)(offsetof(AdjPack<D>, T) - offsetof(AdjPack<D>, X));
}
template <int D>
constexpr uint32_t adj_walk_copy_bytes() {
  return adj_walk_head_bytes<D>() + (uint32_t)(kChunk * kAdjWalkRows * 2) +
         adj_walk_xtb_bytes<D>();
}

template <int D>
struct AdjWalkSmem {
  alignas(128) AdjWalkBuf<D> buf[2];
  float4 xch[kAdjWalkPairs][2][8][32];  // each warp's half of mu K^T, [n8 tile][lane]
  uint64_t bar[2];
};

// The accumulator-layout rows r0 .. r0 + 15, columns c0 .. c0 + 8 NT - 1 of a
// D x D row-major matrix (load; store with lanes t and t^1 swapping halves so
// that every lane writes one 16-byte run).
template <int D, int NT>
__device__ __forceinline__ void sacc_load_cols(float (&sacc)[NT][4], const float* S, int r0, int c0) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int n = 0; n < NT; n++)
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      const float2 x = *reinterpret_cast<const float2*>(S + (size_t)(r0 + gq + 8 * hf) * D + c0 +
                                                        8 * n + 2 * tq);
      sacc[n][2 * hf] = x.x;
      sacc[n][2 * hf + 1] = x.y;
    }
}
template <int D, int NT>
__device__ __forceinline__ void sacc_store_cols(const float (&sacc)[NT][4], float* S, int r0, int c0) {
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3, odd = tq & 1;
#pragma unroll
  for (int n = 0; n < NT; n++) {
    const float s0 = odd ? sacc[n][0] : sacc[n][2];
    const float s1 = odd ? sacc[n][1] : sacc[n][3];
    const float r0v = __shfl_xor_sync(kFull, s0, 1);
    const float r1v = __shfl_xor_sync(kFull, s1, 1);
    float4 out;
    if (!odd) out = make_float4(sacc[n][0], sacc[n][1], r0v, r1v);
    else out = make_float4(r0v, r1v, sacc[n][2], sacc[n][3]);
    const int row = r0 + gq + 8 * odd, col = c0 + 8 * n + 2 * (tq & 2);
    *reinterpret_cast<float4*>(S + (size_t)row * D + col) = out;
  }
}

__device__ __forceinline__ void pair_sync(int id) {
  asm volatile("bar.sync %0, 64;\n" ::"r"(id) : "memory");
}

// One reverse step on a warp's 16 state rows and D / 2 columns (sacc,
// accumulator layout; ch = 0 or 1 the column half):
//   Ydv = (mu K^T) diag(dvec)  (the pair's halves of the contraction added
//         through shared memory; each warp writes half of its tokens to
//         ydv_rows, [row][t])
//   mu <- gamma mu + (-Ydv) Tb K + DO^T X       (this warp's columns)
// rl is the pair's first row within the block (its do columns in DOr).
template <int D>
__device__ __forceinline__ void adj_walk_warp(float (&sacc)[D / 16][4], const AdjWalkBuf<D>& pk,
                                              int rl, int ch, float4 (*xs)[32],
                                              const float4 (*xo)[32], int bar_id,
                                              float* ydv_rows) {
  constexpr int C = kChunk, KH = D / 32;  // k16 steps (and n16 pairs) of a column half
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  using P33 = SplitPairs<kAdjNT, kAdjNT>;
  using P31 = SplitPairs<kAdjNT, 1>;
  using P13 = SplitPairs<1, kAdjNT>;
  float y[8][4];
#pragma unroll
  for (int n = 0; n < 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) y[n][e] = 0.f;
#pragma unroll
  for (int kl = 0; kl < KH; kl++) {
    uint32_t a[kAdjNT][4];
    acc_to_afrag<kAdjNT>(sacc[2 * kl], sacc[2 * kl + 1], a);
#pragma unroll
    for (int np = 0; np < 4; np++) {
      uint32_t b[4];
      ldsm_x4(b, bfrag_nk_addr(pk.K[0], 16 * np, 16 * (KH * ch + kl)));
#pragma unroll
      for (int p = 0; p < P31::kCount; p++) {
        mma16816(y[2 * np], a[P31::a(p)], b[0], b[1]);
        mma16816(y[2 * np + 1], a[P31::a(p)], b[2], b[3]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < 8; n++) xs[n][lane] = make_float4(y[n][0], y[n][1], y[n][2], y[n][3]);
  pair_sync(bar_id);
#pragma unroll
  for (int n = 0; n < 8; n++) {
    const float4 o = xo[n][lane];
    y[n][0] = __fadd_rn(y[n][0], o.x);
    y[n][1] = __fadd_rn(y[n][1], o.y);
    y[n][2] = __fadd_rn(y[n][2], o.z);
    y[n][3] = __fadd_rn(y[n][3], o.w);
  }
#pragma unroll
  for (int n = 0; n < 8; n++) {
    const int t = 8 * n + 2 * tq;
    const float d0 = pk.dvec[t], d1 = pk.dvec[t + 1];
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      y[n][2 * hf] = __fmul_rn(d0, y[n][2 * hf]);
      y[n][2 * hf + 1] = __fmul_rn(d1, y[n][2 * hf + 1]);
      if ((n >> 2) == ch)
        *reinterpret_cast<float2*>(ydv_rows + (size_t)(gq + 8 * hf) * C + t) =
            f2(y[n][2 * hf], y[n][2 * hf + 1]);
    }
  }
  // Z = (-Ydv) Tb, the full 16 x C on both warps of the pair (splitting it
  // between them costs a second exchange and was slower)
  float z[8][4];
#pragma unroll
  for (int n = 0; n < 8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) z[n][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    float n0[4], n1[4];
#pragma unroll
    for (int e = 0; e < 4; e++) {
      n0[e] = -y[2 * ks][e];
      n1[e] = -y[2 * ks + 1][e];
    }
    uint32_t a[kAdjNT][4];
    acc_to_afrag<kAdjNT>(n0, n1, a);
#pragma unroll
    for (int np = 0; np < 4; np++) {
      if (np > ks) continue;
      uint32_t b[kAdjNT][4];
#pragma unroll
      for (int qq = 0; qq < kAdjNT; qq++)
        ldsm_x4_t(b[qq], bfrag_kn_addr(pk.Tb[qq], 16 * ks, 16 * np));
#pragma unroll
      for (int p = 0; p < P33::kCount; p++) {
        mma16816(z[2 * np], a[P33::a(p)], b[P33::b(p)][0], b[P33::b(p)][1]);
        mma16816(z[2 * np + 1], a[P33::a(p)], b[P33::b(p)][2], b[P33::b(p)][3]);
      }
    }
  }
  // mu <- gamma mu, then + Z K, then + DO^T X (this warp's columns)
  const float gam = pk.gamma[0];
#pragma unroll
  for (int n = 0; n < D / 16; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) sacc[n][e] = __fmul_rn(gam, sacc[n][e]);
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    uint32_t a[kAdjNT][4];
    acc_to_afrag<kAdjNT>(z[2 * ks], z[2 * ks + 1], a);
#pragma unroll
    for (int np = 0; np < KH; np++) {
      uint32_t b[4];
      ldsm_x4_t(b, bfrag_kn_addr(pk.K[0], 16 * ks, 16 * (KH * ch + np)));
#pragma unroll
      for (int p = 0; p < P31::kCount; p++) {
        mma16816(sacc[2 * np], a[P31::a(p)], b[0], b[1]);
        mma16816(sacc[2 * np + 1], a[P31::a(p)], b[2], b[3]);
      }
    }
  }
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    uint32_t a[1][4];
    ldsm_x4_t(a[0], afrag_t_addr(pk.DOr[0], rl, 16 * ks));
#pragma unroll
    for (int np = 0; np < KH; np++) {
      uint32_t b[kAdjNT][4];
#pragma unroll
      for (int qq = 0; qq < kAdjNT; qq++)
        ldsm_x4_t(b[qq], bfrag_kn_addr(pk.X[qq], 16 * ks, 16 * (KH * ch + np)));
#pragma unroll
      for (int p = 0; p < P13::kCount; p++) {
        mma16816(sacc[2 * np], a[P13::a(p)], b[P13::b(p)][0], b[P13::b(p)][1]);
        mma16816(sacc[2 * np + 1], a[P13::a(p)], b[P13::b(p)][2], b[P13::b(p)][3]);
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kAdjWalkThreads, 1)
    k_adj_walk(const int32_t* __restrict__ cu, int H, int32_t* __restrict__ hdr,
               const int32_t* __restrict__ chunk_off, const int32_t* __restrict__ seq_order,
               const char* __restrict__ apacks,
               const float* __restrict__ ds_final, float* __restrict__ mu_end,
               float* __restrict__ ydv, float* __restrict__ d_h0,
               const __grid_constant__ CUtensorMap map_do) {
  constexpr int C = kChunk, RB = D / kAdjWalkRows, NT = D / 16;
  static_assert(D % kAdjWalkRows == 0, "whole row blocks");
  constexpr uint32_t HB = adj_walk_head_bytes<D>(), XB = adj_walk_xtb_bytes<D>();
  constexpr uint32_t DB = (uint32_t)(C * kAdjWalkRows * 2);
  static_assert(HB % 16 == 0 && XB % 16 == 0 && DB % 16 == 0 &&
                    offsetof(AdjWalkBuf<D>, DOr) % 128 == 0 && sizeof(AdjWalkBuf<D>) % 128 == 0 &&
                    offsetof(AdjWalkBuf<D>, K) == offsetof(AdjPack<D>, K) &&
                    offsetof(AdjWalkBuf<D>, X) % 16 == 0 &&
                    offsetof(AdjWalkBuf<D>, Tb) - offsetof(AdjWalkBuf<D>, X) ==
                        offsetof(AdjPack<D>, Tb) - offsetof(AdjPack<D>, X),
                "bulk copies of 16-byte pieces into matching layouts");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AdjWalkSmem<D>& sm = *reinterpret_cast<AdjWalkSmem<D>*>(smem_raw);
  pdl_wait();  // the adjoint prep's packs
  pdl_trigger();
  if (hdr[kHdrValid] != 1) return;
  // Blocks go out sequence by sequence, most chunks first (the chunk table's
  // order), so that the longest serial chains start in the first wave.
  const int per_seq = H * RB;
  const int n = seq_order[blockIdx.x / per_seq];
  const int h = (blockIdx.x % per_seq) / RB, rb = blockIdx.x % RB, t = threadIdx.x;
  const int w = t >> 5, pair = w >> 1, ch = w & 1;
  const int rl = 16 * pair, r0 = kAdjWalkRows * rb + rl, c0 = (D / 2) * ch;
  const size_t DD = (size_t)D * D;
  const int64_t L = (int64_t)cu[n + 1] - cu[n];
  const int64_t nc = (L + C - 1) / C;
  const int64_t base = chunk_off[n];
  auto pack = [&](int64_t cc) {
    return apacks + ((size_t)(base + cc) * H + h) * adj_pack_bytes<D>();
  };
  // The block's do columns, core-layout column groups R rb .. R rb + R - 1
  // (R = kAdjWalkRows / 8) of the chunk's do plane, come from the input by
  // one tensor-map copy.
  const int tok0 = cu[n];
  auto fetch = [&](int b, int64_t cc) {
    const uint32_t mb = smem_u32(&sm.bar[b]);
    const char* src = pack(cc);
    mbar_expect_tx(mb, HB + DB + XB);
    bulk_load(smem_u32(&sm.buf[b]), src, HB, mb);
    tma_load_4d(smem_u32(sm.buf[b].DOr[0]), &map_do, 0, tok0 + (int)cc * C,
                (kAdjWalkRows / 8) * rb, h, mb);
    bulk_load(smem_u32(sm.buf[b].X[0]), src + offsetof(AdjPack<D>, X), XB, mb);
  };
  pack_bars_init(sm.bar);
  float sacc[NT][4];
  if (ds_final) {
    sacc_load_cols<D, NT>(sacc, ds_final + ((size_t)n * H + h) * DD, r0, c0);
  } else {
#pragma unroll
    for (int i = 0; i < NT; i++)
#pragma unroll
      for (int e = 0; e < 4; e++) sacc[i][e] = 0.f;
  }
  if (t == 0 && nc > 0) fetch(0, nc - 1);
  int64_t issued = nc > 0 ? 1 : 0;
  bool ok = true;
  for (int64_t j = 0; j < nc; j++) {
    const int64_t cc = nc - 1 - j;
    if (cc >= 1) {
      if (t == 0) fetch((int)((j + 1) & 1), cc - 1);
      issued = j + 2;
    }
    const size_t unit = (size_t)(base + cc) * H + h;
    sacc_store_cols<D, NT>(sacc, mu_end + unit * DD, r0, c0);
    if (__syncthreads_or(!pack_wait(sm.bar, j))) {
      ok = false;
      pack_drain(sm.bar, j, issued);
      break;
    }
    if (j == 0 && L % C != 0) {
      // The trailing partial chunk: its do rows past the sequence's end are
      // the next sequence's tokens (or zeros past T); they must be zero.
      const int len = (int)(L % C);
      __nv_bfloat16* dor = sm.buf[0].DOr[0];
      for (int e = t; e < (kAdjWalkRows / 8) * (C - len); e += kAdjWalkThreads) {
        const int grp = e / (C - len), r = len + e % (C - len);
        *reinterpret_cast<uint4*>(dor + (grp * C + r) * 8) = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncthreads();
    }
    adj_walk_warp<D>(sacc, sm.buf[j & 1], rl, ch, sm.xch[pair][ch], sm.xch[pair][ch ^ 1],
                     1 + pair, ydv + (unit * D + r0) * C);
    __syncthreads();  // buffer j & 1 is refilled with chunk cc - 2; xch is free
  }
  if (!ok) {
    if (t == 0) atomicOr(&hdr[kHdrError], kErrTimeout);
    return;
  }
  if (d_h0) sacc_store_cols<D, NT>(sacc, d_h0 + ((size_t)n * H + h) * DD, r0, c0);
}

// ----------------------------------------------------------------------------
// The W solve (one (chunk, head) per block)
// ----------------------------------------------------------------------------
constexpr int kAdjWThreads = 256;

template <int D>
struct AdjWSmem {
  float dvec[kChunk];
  float beta[kChunk];
  float gamma[4];
  alignas(128) __nv_bfloat16 DO[1][kChunk * D];    // [r][i], a tensor-map destination
  __nv_bfloat16 T[kAdjNT][kChunk * kChunk];        // [m][t]
  __nv_bfloat16 Pm[kAdjNT][kChunk * kChunk];       // [r][t]
  __nv_bfloat16 R[kAdjNT][kChunk * D];             // right-hand side, [m][i]
  uint64_t bar;                                    // the do copy's completion
};
// cp.async pieces and ldmatrix rows are 16-byte aligned in every plane.
static_assert(offsetof(AdjWSmem<128>, T) % 16 == 0 && offsetof(AdjWSmem<128>, Pm) % 16 == 0 &&
                  offsetof(AdjWSmem<128>, R) % 16 == 0 && offsetof(AdjWSmem<64>, T) % 16 == 0 &&
                  offsetof(AdjWSmem<64>, R) % 16 == 0,
              "16-byte aligned planes");

// The W solve of one (chunk, head) item; one block of kAdjWThreads threads.
template <int D>
__device__ __forceinline__ void adj_w_item(AdjWSmem<D>& sm, int c, int h,
                                           const int32_t* __restrict__ cu, int H, float scale,
                                           const int32_t* __restrict__ chunk_off,
                                           const int32_t* __restrict__ chunk_seq,
                                           const char* __restrict__ apacks,
                                           const CUtensorMap* map_do, int32_t* __restrict__ error,
                                           const float* __restrict__ ydv, float* __restrict__ wbuf,
                                           float* __restrict__ d_v) {
  using bf16 = __nv_bfloat16;
  constexpr int C = kChunk, PL = C * C, PD = C * D, NT8 = D / 16;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const int mt = w & 3, nh = w >> 2;
  const FillItem it = fill_item(c * H + h, H, cu, chunk_off, chunk_seq);
  const int len = it.len;
  const size_t tb = (size_t)it.t0 * H + h;
  const AdjPack<D>& pk =
      *reinterpret_cast<const AdjPack<D>*>(apacks + ((size_t)c * H + h) * adj_pack_bytes<D>());
  // The chunk's do rows from the input by one tensor-map copy (rows past its
  // length zeroed once it lands); the pack's head, T and Pm terms by
  // cp.async (16-byte pieces).
  const uint32_t bar = smem_u32(&sm.bar);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_expect_tx(bar, (uint32_t)PD * 2);
    tma_load_4d(smem_u32(sm.DO[0]), map_do, 0, (int)it.t0, 0, h, bar);
  }
  for (int e = tid; e < (int)(2 * C + 4) / 4; e += kAdjWThreads)
    cp_async16(reinterpret_cast<float4*>(sm.dvec) + e, reinterpret_cast<const float4*>(pk.dvec) + e);
  for (int e = tid; e < 2 * kAdjNT * PL / 8; e += kAdjWThreads)
    cp_async16(reinterpret_cast<uint4*>(sm.T[0]) + e, reinterpret_cast<const uint4*>(pk.T[0]) + e);
  cp_async_commit();
  cp_async_wait<0>();
  const bool ok = mbar_wait(bar, 0, kTcWaitPolls);
  if (ok && len < C) {
    for (int e = tid; e < (D / 8) * (C - len); e += kAdjWThreads) {
      const int grp = e / (C - len), r = len + e % (C - len);
      *reinterpret_cast<uint4*>(&sm.DO[0][(grp * C + r) * 8]) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (__syncthreads_or(!ok)) {  // the do rows never arrived: wait once more and stop
    if (tid == 0) atomicOr(error, kErrTimeout);
    (void)mbar_wait(bar, 0, kTcWaitPolls);
    return;
  }

  using P33 = SplitPairs<kAdjNT, kAdjNT>;
  using P31 = SplitPairs<kAdjNT, 1>;
  // R = Ydv^T + scale Pm^T DO on warp (mt, nh)'s tile: tokens 16 mt .., rows
  // i = (D / 2) nh .. (Pm^T[t][r] = Pm[r][t] vanishes for r < t).
  float acc[NT8][4];
#pragma unroll
  for (int n = 0; n < NT8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) acc[n][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    if (ks < mt) continue;
    uint32_t a[kAdjNT][4];
#pragma unroll
    for (int qq = 0; qq < kAdjNT; qq++) ldsm_x4_t(a[qq], afrag_t_addr(sm.Pm[qq], 16 * mt, 16 * ks));
#pragma unroll
    for (int np = 0; np < NT8 / 2; np++) {
      uint32_t b[4];
      ldsm_x4_t(b, bfrag_kn_addr(sm.DO[0], 16 * ks, (D / 2) * nh + 16 * np));
#pragma unroll
      for (int p = 0; p < P31::kCount; p++) {
        mma16816(acc[2 * np], a[P31::a(p)], b[0], b[1]);
        mma16816(acc[2 * np + 1], a[P31::a(p)], b[2], b[3]);
      }
    }
  }
  const float* yd = ydv + ((size_t)c * H + h) * D * C;
#pragma unroll
  for (int n = 0; n < NT8; n++)
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      const int m = 16 * mt + gq + 8 * hf, i = (D / 2) * nh + 8 * n + 2 * tq;
      const float r0v = __fmaf_rn(scale, acc[n][2 * hf], yd[(size_t)i * C + m]);
      const float r1v = __fmaf_rn(scale, acc[n][2 * hf + 1], yd[(size_t)(i + 1) * C + m]);
      put3(sm.R[0], PD, core_off<C>(m, i), r0v, r1v);
    }
  __syncthreads();
  // W = T^T R (T^T[t][m] = T[m][t] vanishes for m < t).
#pragma unroll
  for (int n = 0; n < NT8; n++)
#pragma unroll
    for (int e = 0; e < 4; e++) acc[n][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ks++) {
    if (ks < mt) continue;
    uint32_t a[kAdjNT][4];
#pragma unroll
    for (int qq = 0; qq < kAdjNT; qq++) ldsm_x4_t(a[qq], afrag_t_addr(sm.T[qq], 16 * mt, 16 * ks));
#pragma unroll
    for (int np = 0; np < NT8 / 2; np++) {
      uint32_t b[kAdjNT][4];
#pragma unroll
      for (int qq = 0; qq < kAdjNT; qq++)
        ldsm_x4_t(b[qq], bfrag_kn_addr(sm.R[qq], 16 * ks, (D / 2) * nh + 16 * np));
#pragma unroll
      for (int p = 0; p < P33::kCount; p++) {
        mma16816(acc[2 * np], a[P33::a(p)], b[P33::b(p)][0], b[P33::b(p)][1]);
        mma16816(acc[2 * np + 1], a[P33::a(p)], b[P33::b(p)][2], b[P33::b(p)][3]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NT8; n++)
#pragma unroll
    for (int hf = 0; hf < 2; hf++) {
      const int t = 16 * mt + gq + 8 * hf;
      if (t >= len) continue;
      const int i = (D / 2) * nh + 8 * n + 2 * tq;
      const size_t o = (tb + (size_t)t * H) * D + i;
      const float bt = sm.beta[t];
      *reinterpret_cast<float2*>(wbuf + o) = f2(acc[n][2 * hf], acc[n][2 * hf + 1]);
      *reinterpret_cast<float2*>(d_v + o) =
          f2(__fmul_rn(bt, acc[n][2 * hf]), __fmul_rn(bt, acc[n][2 * hf + 1]));
    }
}

}  // namespace gdn
