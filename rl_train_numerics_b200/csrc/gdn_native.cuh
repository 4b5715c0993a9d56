// gdn_native.cuh -- outputs of the chunked ("native mixed") forward on the
// fifth-generation tensor cores, d = 128 with bf16 inputs.
//
// "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
// section "Solving the linear-attention headache": the per-layer table's
// first column is the usual layout, whose training and prefill evaluate the
// layer chunkwise in parallel (the UT / WY form) while decode runs the
// per-token recurrence, so that prefill and decode round differently.  Its
// chunkwise outputs, from the state S entering a chunk (chunk-local tokens
// i, j; G the chunk's cumulative log-decay; U as in gdn_boundary.cuh):
//
//   S_i = e^{G_i} S + sum_{j <= i} e^{G_i - G_j} u_j k_j^T
//   o_i = scale * (e^{G_i} S q_i + sum_{j <= i} e^{G_i - G_j} (q_i . k_j) u_j)
//   U   = Tv V - Tb (K S^T)
//
// i.e. with Pm_ij = [j <= i] e^{G_i - G_j} (q_i . k_j),
//   O^T = (S Q^T) diag(e^G) + U^T Pm^T        (rows: value channels).
// The states entering the chunks come from the CPR forward's first pass (the
// same boundary prep and walk); this file adds the output products.  One
// block of 512 threads per SM takes (chunk, head) items in turn; tensor
// memory (512 columns, fp32 accumulators; bf16 terms two per column):
//   [  0,128)  S terms (the A operand of Y and Oa); then P (final state)
//   [128,192)  Y; then the -Y terms; then the U^T terms (A of Ob)
//   [192,256)  Z = U^T
//   [256,320)  Oa = S Q^T
//   [320,384)  Ob = U^T Pm^T
//   [384,448)  Ud terms (A of P, for a sequence's trailing partial chunk)
// Rounds of products (warp 0 issues; one mbarrier):
//   1  Y = S K^T, Oa = S Q^T, Z = V^T Tv^T        meanwhile: Pm (mma.sync)
//   2  Z -= Y Tb^T                                (as in the boundary walk)
//   3  Ob = Z Pm^T; for a trailing partial chunk also P = Ud K
// then o_i = scale * fma(e^{G_i}, Oa, Ob) per element, and for a trailing
// partial chunk the final state exp(G) S + P (the chunk is prepared
// zero-padded: its padding tokens are identity steps).  Operands that are not
// exact in bf16 (S, Y, Z, Tb, Tv, Pm) are split into two bf16 terms and the
// products of the term pairs (hi, hi), (hi, lo), (lo, hi) accumulate in that
// order.  Every wait is bounded.
#pragma once

#include "gdn_boundary.cuh"
#include "gdn_fill.cuh"

namespace gdn {

constexpr uint32_t kNtSA = 0, kNtP = 0, kNtY = 128, kNtYA = 128, kNtZ = 192, kNtOa = 256,
                   kNtOb = 320, kNtUd = 384;
constexpr uint32_t kNtCols = 512;
constexpr int kNtThreads = 512;  // 16 warps: 4 lane quadrants x 4 column slices
constexpr int kNtPmWarp0 = 6;    // warps 6 .. 15 form Pm, one 16 x 16 block each

struct NativeSmem {
  WalkPack<128, __nv_bfloat16> buf[2];
  alignas(128) __nv_bfloat16 Q[1][kChunk * 128];     // queries, core layout (K-major)
  alignas(128) __nv_bfloat16 Pm[2][kChunk * kChunk];  // Pm terms, core layout rows i, cols j
  double G[kChunk];
  float eG[kChunk];
  float graw[kChunk];
  uint64_t ld_bar[2];
  uint64_t mbar;
  uint32_t tmem;
};

// (m-tile, n-tile) of Pm block b = 0 .. 9, the lower triangle of 4 x 4.
__device__ __forceinline__ void pm_block(int b, int& mt, int& nt) {
  mt = b < 1 ? 0 : b < 3 ? 1 : b < 6 ? 2 : 3;
  nt = b - (mt * (mt + 1)) / 2;
}

template <class OUT>
__global__ void __launch_bounds__(kNtThreads, 1)
    k_native_tc(const __nv_bfloat16* __restrict__ q, const float* __restrict__ g,
                const int32_t* __restrict__ cu, int H, float scale, int32_t* __restrict__ hdr,
                const int32_t* __restrict__ chunk_off, const int32_t* __restrict__ chunk_seq,
                const char* __restrict__ packs, const float* __restrict__ bstate,
                OUT* __restrict__ o, float* __restrict__ s_final) {
  using bf16 = __nv_bfloat16;
  constexpr int D = 128, SC = D / 4, YC = kChunk / 4;
  constexpr size_t PB = pack_size<D, bf16>();
  constexpr uint32_t TPLANE = kChunk * kChunk * 2;
  constexpr uint32_t IY = idesc_bf16(kTcRows, kChunk, false, false);
  constexpr uint32_t IP = idesc_bf16(kTcRows, D, false, true);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  NativeSmem& sm = *reinterpret_cast<NativeSmem*>(smem_raw);
  if (hdr[kHdrValid] != 1) return;
  const int n_items = hdr[kHdrChunks] * H;
  if ((int)blockIdx.x >= n_items) return;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31, cs = w >> 2;
  const int row = 32 * (w & 3) + lane;
  const size_t DD = (size_t)D * D;
  pack_bars_init(sm.ld_bar);
  TcCtx cx;
  tc_setup(cx, &sm.mbar, &sm.tmem, kNtCols);
  const uint32_t tl = cx.tmem + ((uint32_t)(32 * (w & 3)) << 16);  // this warp's lanes
  const uint32_t qb = smem_u32(sm.Q[0]), pmb = smem_u32(sm.Pm[0]);
  auto pack_of = [&](int item) { return packs + (size_t)item * PB; };
  if (t == 0) pack_fetch<D, bf16>(sm.buf[0], pack_of(blockIdx.x), &sm.ld_bar[0]);
  int64_t j = 0, issued = 1;
  int status = kStepDone;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, j++) {
    const int next = item + (int)gridDim.x;
    const FillItem it = fill_item(item, H, cu, chunk_off, chunk_seq);
    const size_t tb = (size_t)it.t0 * H + it.h;
    const int64_t nc = (it.L + kChunk - 1) / kChunk;
    const bool fin = it.ci == nc - 1 && it.len < kChunk;  // trailing partial chunk
    if (next < n_items) {
      if (t == 0) pack_fetch<D, bf16>(sm.buf[(j + 1) & 1], pack_of(next), &sm.ld_bar[(j + 1) & 1]);
      issued = j + 2;
      const FillItem nx = fill_item(next, H, cu, chunk_off, chunk_seq);
      if (t == 32) prefetch_l2(bstate + ((size_t)nx.c * H + nx.h) * DD, (uint32_t)(DD * 4));
      if (t >= 64 && t < 64 + nx.len)
        prefetch_l2(q + ((size_t)(nx.t0 + (t - 64)) * H + nx.h) * D, (uint32_t)(D * 2));
    }
    // This item's queries (zero past its length), gates and entering state.
    stage_planes<D, bf16>(sm.Q, q + tb * D, (size_t)H * D, kNtThreads, it.len);
    cp_async_commit();
    if (t < kChunk) sm.graw[t] = t < it.len ? g[tb + (size_t)t * H] : 0.f;
    float s[SC];
    {
      const float* src = bstate + ((size_t)it.c * H + it.h) * DD + (size_t)row * D;
#pragma unroll
      for (int c = 0; c < SC; c += 4) {
        const float4 x = ld4(src + bst_col(row, cs * SC + c));
        s[c] = x.x, s[c + 1] = x.y, s[c + 2] = x.z, s[c + 3] = x.w;
      }
    }
    tc_fence_after();
    store_terms<16, false>(tl + kNtSA + (cs * SC) / 2, 64, s);
    tmem_wait_st();
    cp_async_wait<0>();
    fence_async_smem();
    const bool in_ok = pack_wait(sm.ld_bar, j);
    tc_fence_before();
    if (__syncthreads_or(!in_ok)) {
      status = kStepNoInputs;
      break;
    }
    const WalkPack<D, bf16>& pk = sm.buf[j & 1];
    const uint32_t kb = smem_u32(pk.kv.K[0]), vb = smem_u32(pk.kv.V[0]);
    const uint32_t tbb = smem_u32(pk.head.TbT[0]), tvb = smem_u32(pk.head.TvT[0]);
    // First product round
    if (w == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < D / 16; ks++)
#pragma unroll
        for (int a = 0; a < 2; a++)
          umma_bf16_ts(cx.tmem + kNtY, cx.tmem + kNtSA + 64 * a + 8 * ks,
                       desc_kmajor<kChunk>(kb + ks * 2 * kChunk * 16), IY, (ks > 0 || a > 0));
#pragma unroll
      for (int ks = 0; ks < D / 16; ks++)
#pragma unroll
        for (int a = 0; a < 2; a++)
          umma_bf16_ts(cx.tmem + kNtOa, cx.tmem + kNtSA + 64 * a + 8 * ks,
                       desc_kmajor<kChunk>(qb + ks * 2 * kChunk * 16), IY, (ks > 0 || a > 0));
#pragma unroll
      for (int ks = 0; ks < kChunk / 16; ks++)
#pragma unroll
        for (int qq = 0; qq < 2; qq++)
          umma_bf16(cx.tmem + kNtZ + 16 * ks, desc_mnmajor<kChunk>(vb + ks * 256),
                    desc_mnmajor<kChunk>(tvb + qq * TPLANE + ks * 256 + ks * 2 * kChunk * 16),
                    idesc_bf16(kTcRows, kChunk - 16 * ks, true, true), (ks > 0 || qq > 0));
      umma_commit(cx.mbar);
      chunk_cumsum_g(sm.graw, sm.G);
#pragma unroll
      for (int e = 0; e < 2; e++)
        sm.eG[2 * lane + e] = expf(__double2float_rn(sm.G[2 * lane + e]));
    }
    // Meanwhile: Q K^T on the 16 x 16 blocks of the lower triangle.
    float pacc[2][4];
    int mt = 0, nt = 0;
    const bool pm_warp = w >= kNtPmWarp0;
    if (pm_warp) {
      pm_block(w - kNtPmWarp0, mt, nt);
#pragma unroll
      for (int n = 0; n < 2; n++)
#pragma unroll
        for (int e = 0; e < 4; e++) pacc[n][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ks++) {
        uint32_t a[4], b[4];
        ldsm_x4(a, afrag_addr(sm.Q[0], 16 * mt, 16 * ks));
        ldsm_x4(b, bfrag_nk_addr(pk.kv.K[0], 16 * nt, 16 * ks));
        mma16816(pacc[0], a, b[0], b[1]);
        mma16816(pacc[1], a, b[2], b[3]);
      }
    }
    __syncthreads();  // G, e^G ready
    if (pm_warp) {
      const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
      for (int n = 0; n < 2; n++)
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
          const int i = 16 * mt + gq + 8 * hf, jj = 16 * nt + 8 * n + 2 * tq;
          float x[2];
#pragma unroll
          for (int e = 0; e < 2; e++) {
            const int jc = jj + e;
            x[e] = 0.f;
            if (jc <= i && i < it.len)
              x[e] = __fmul_rn(expf(__double2float_rn(sm.G[i] - sm.G[jc])), pacc[n][2 * hf + e]);
          }
          uint32_t hi, lo;
          split2(x[0], x[1], hi, lo);
          *reinterpret_cast<uint32_t*>(&sm.Pm[0][core_off<kChunk>(i, jj)]) = hi;
          *reinterpret_cast<uint32_t*>(&sm.Pm[1][core_off<kChunk>(i, jj)]) = lo;
        }
    }
    bool ok = tc_wait(cx);
    // -Y terms over Y (once every thread has its slice of Y)
    {
      float y[YC];
      tmem_load<YC>(tl + kNtY + cs * YC, y);
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      store_terms<YC / 2, true>(tl + kNtYA + (cs * YC) / 2, 32, y);
      tmem_wait_st();
    }
    fence_async_smem();  // Pm planes, written by the threads, read by the tensor cores
    tc_fence_before();
    if (__syncthreads_or(!ok)) {
      status = kStepFailed;
      break;
    }
    // Second product round: Z -= Y Tb^T
    if (w == 0) {
      tc_fence_after();
      using PY = SplitPairs<2, 2>;
#pragma unroll
      for (int ks = 0; ks < kChunk / 16; ks++)
#pragma unroll
        for (int p = 0; p < PY::kCount; p++)
          umma_bf16_ts(cx.tmem + kNtZ + 16 * ks, cx.tmem + kNtYA + 32 * PY::a(p) + 8 * ks,
                       desc_mnmajor<kChunk>(tbb + PY::b(p) * TPLANE + ks * 256 + ks * 2 * kChunk * 16),
                       idesc_bf16(kTcRows, kChunk - 16 * ks, false, true), 1u);
      umma_commit(cx.mbar);
    }
    ok = tc_wait(cx);
    // U^T terms (A of Ob) and, for a trailing partial chunk, Ud terms
    {
      float z[YC];
      tmem_load<YC>(tl + kNtZ + cs * YC, z);
      store_terms<YC / 2, false>(tl + kNtYA + (cs * YC) / 2, 32, z);
      if (fin) {
#pragma unroll
        for (int i = 0; i < YC; i++) z[i] = __fmul_rn(pk.head.dvec[cs * YC + i], z[i]);
        store_terms<YC / 2, false>(tl + kNtUd + (cs * YC) / 2, 32, z);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    if (__syncthreads_or(!ok)) {
      status = kStepFailed;
      break;
    }
    // Third product round: Ob = Z Pm^T (Pm lower triangular: k16 step ks reaches the
    // columns i >= 16 ks); P = Ud K for a trailing partial chunk
    if (w == 0) {
      tc_fence_after();
      using PY = SplitPairs<2, 2>;
#pragma unroll
      for (int ks = 0; ks < kChunk / 16; ks++)
#pragma unroll
        for (int p = 0; p < PY::kCount; p++)
          umma_bf16_ts(cx.tmem + kNtOb + 16 * ks, cx.tmem + kNtYA + 32 * PY::a(p) + 8 * ks,
                       desc_kmajor<kChunk>(pmb + PY::b(p) * TPLANE + ks * 2 * kChunk * 16 + ks * 256),
                       idesc_bf16(kTcRows, kChunk - 16 * ks, false, false), (ks > 0 || p > 0));
      if (fin) {
#pragma unroll
        for (int ks = 0; ks < kChunk / 16; ks++)
#pragma unroll
          for (int a = 0; a < 2; a++)
            umma_bf16_ts(cx.tmem + kNtP, cx.tmem + kNtUd + 32 * a + 8 * ks,
                         desc_mnmajor<kChunk>(kb + ks * 256), IP, (ks > 0 || a > 0));
      }
      umma_commit(cx.mbar);
    }
    ok = tc_wait(cx);
    if (ok) {
      float oa[YC], obv[YC];
      tmem_load<YC>(tl + kNtOa + cs * YC, oa);
      tmem_load<YC>(tl + kNtOb + cs * YC, obv);
      OUT* op = o + tb * D + row;
#pragma unroll
      for (int i = 0; i < YC; i++) {
        const int tok = cs * YC + i;
        if (tok < it.len)
          st1(op + (size_t)tok * H * D,
              __fmul_rn(scale, __fmaf_rn(sm.eG[tok], oa[i], obv[i])));
      }
      if (fin && s_final) {
        const float gam = pk.head.gamma[0];
        float* dst = s_final + ((size_t)it.n * H + it.h) * DD + (size_t)row * D + cs * SC;
        float pv[32];
        tmem_load<32>(tl + kNtP + cs * SC, pv);
#pragma unroll
        for (int c = 0; c < SC; c += 4)
          *reinterpret_cast<float4*>(dst + c) =
              make_float4(__fmaf_rn(gam, s[c], pv[c]), __fmaf_rn(gam, s[c + 1], pv[c + 1]),
                          __fmaf_rn(gam, s[c + 2], pv[c + 2]), __fmaf_rn(gam, s[c + 3], pv[c + 3]));
      }
    }
    tc_fence_before();
    if (__syncthreads_or(!ok)) {
      status = kStepFailed;
      break;
    }
  }
  if (status != kStepDone) {
    pack_drain(sm.ld_bar, j, issued);
    if (status == kStepFailed) tc_drain(cx);
    if (t == 0) atomicOr(&hdr[kHdrError], kErrTimeout);
  }
  tc_teardown(cx, kNtCols);
}

}  // namespace gdn
