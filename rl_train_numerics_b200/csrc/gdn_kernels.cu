// gdn_kernels.cu -- CUDA kernels of the CPR Gated DeltaNet layer (sm_100a).
//
// Forward ("NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI
// Training Runs", section "Solving the linear-attention headache"): two
// passes, the states at the chunk edges first, then every chunk's tokens
// from its entry state:
//   k_chunk_table   one block: validates cu_seqlens, numbers the chunks,
//                   orders the sequences by chunk count
//   k_prep          one block per (chunk, head): boundary prep of full chunks
//   k_walk          one block per (sequence, head): serial walk (mma.sync,
//                   d = 64)
//   k_walk_tc       the same on tcgen05 / tensor memory (d = 128, bf16)
//   k_fill          persistent blocks over (chunk, head) items: per-token
//                   recurrence from each chunk's boundary state
// Decode (same section: the recurrent form re-synchronised every chunk):
//   k_dec_step      one block per (row, head): one recurrence step; units
//                   whose chunk buffer became full go on a work list
//   k_resync        persistent blocks: the chunk boundary of listed units
//   k_bnd           one block per (row, head): gdn_chunk_boundary
//   k_handoff       prefill -> decode state
#include <cuda.h>
#include <string.h>

#include "gdn_boundary.cuh"
#include "gdn_fill.cuh"
#include "gdn_layout.h"
#include "gdn_native.cuh"
#include "gdn_tmap.h"

namespace gdn {

// ----------------------------------------------------------------------------
// Chunk table
// ----------------------------------------------------------------------------
constexpr int kTableThreads = 256;
constexpr int kTableWarps = kTableThreads / 32;  // at most 32

__global__ void __launch_bounds__(kTableThreads)
    k_chunk_table(const int32_t* __restrict__ cu, int N, int64_t T, int H, int32_t* hdr,
                  int32_t* chunk_off, int32_t* seq_order, int32_t* chunk_seq,
                  int32_t* fill_off, int64_t max_chunks) {
  __shared__ long long part[64 + kTableThreads];
  __shared__ int bucket[kTableThreads];
  __shared__ int bad;
  pdl_trigger();
  const int tid = threadIdx.x;
  if (tid == 0) bad = (cu[0] != 0 || (int64_t)cu[N] != T) ? 1 : 0;
  __syncthreads();
  const int64_t per = ((int64_t)N + kTableThreads - 1) / kTableThreads;
  const int64_t n0 = min((int64_t)N, (int64_t)tid * per);
  const int64_t n1 = min((int64_t)N, n0 + per);
  long long local = 0;
  int mybad = 0;
  for (int64_t n = n0; n < n1; n++) {
    const int64_t L = (int64_t)cu[n + 1] - (int64_t)cu[n];
    if (L < 0) mybad = 1;
    else local += (L + kChunk - 1) / kChunk;
  }
  if (mybad) atomicOr(&bad, 1);
  // Exclusive prefix sum of the per-thread chunk counts: inclusive scans
  // inside each warp, then over the warp totals.
  const int lane = tid & 31, warp = tid >> 5;
  long long x = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long y = __shfl_up_sync(kFull, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) part[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long wsum = lane < kTableWarps ? part[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(kFull, wsum, off);
      if (lane >= off) wsum += y;
    }
    part[32 + lane] = wsum;  // inclusive over warps 0 .. lane
  }
  __syncthreads();
  const long long run = part[32 + kTableWarps - 1];
  part[64 + tid] = x - local + (warp > 0 ? part[32 + warp - 1] : 0);  // exclusive, this thread
  if (tid == 0) {
    if (run > max_chunks) bad = 1;
    hdr[kHdrChunks] = bad ? 0 : (int32_t)run;
    hdr[kHdrFillNext] = 0;
    hdr[kHdrFill0Next] = 0;
    if (!bad) chunk_off[N] = (int32_t)run;
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      atomicOr(&hdr[kHdrError], kErrCuSeqlens);
      hdr[kHdrValid] = 0;
    }
    return;
  }
  long long off = part[64 + tid];
  for (int64_t n = n0; n < n1; n++) {
    const int64_t L = (int64_t)cu[n + 1] - (int64_t)cu[n];
    const long long nc = (L + kChunk - 1) / kChunk;
    chunk_off[n] = (int32_t)off;
    for (long long i = 0; i < nc; i++) chunk_seq[off + i] = (int32_t)n;
    off += nc;
  }
  // The sequences by chunk count, most first (counts from kTableThreads - 1
  // up share one place): the order in which serial per-sequence passes
  // launch their blocks, so that the longest chains start in the first wave.
  // Equal counts land in any order; no result depends on it.
  bucket[tid] = 0;
  __syncthreads();
  auto key = [&](int64_t n) {
    const int64_t nc = ((int64_t)cu[n + 1] - (int64_t)cu[n] + kChunk - 1) / kChunk;
    return (int)min(nc, (int64_t)kTableThreads - 1);
  };
  for (int64_t n = n0; n < n1; n++) atomicAdd(&bucket[key(n)], 1);
  __syncthreads();
  {
    // Exclusive scan in descending key order: thread tid takes key
    // kTableThreads - 1 - tid.
    const int mine = bucket[kTableThreads - 1 - tid];
    int xs = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, xs, o);
      if (lane >= o) xs += y;
    }
    if (lane == 31) part[warp] = xs;
    __syncthreads();
    if (warp == 0) {
      long long ws = lane < kTableWarps ? part[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(kFull, ws, o);
        if (lane >= o) ws += y;
      }
      part[32 + lane] = ws;
    }
    __syncthreads();
    bucket[kTableThreads - 1 - tid] = xs - mine + (warp > 0 ? (int)part[32 + warp - 1] : 0);
  }
  __syncthreads();
  for (int64_t n = n0; n < n1; n++) seq_order[atomicAdd(&bucket[key(n)], 1)] = (int32_t)n;
  __syncthreads();  // seq_order complete
  // The fill order: every chunk after a sequence's first, the sequences in
  // seq_order reversed (fewest chunks first: their walks end first), chunks
  // ascending within a sequence.  Here each sequence's first entry
  // (exclusive scan of the per-thread entry counts as above); the prep's
  // blocks write the entries.
  {
    long long mine = 0;
    for (int64_t r = n0; r < n1; r++) {
      const int sq = seq_order[N - 1 - r];
      const long long nc = chunk_off[sq + 1] - chunk_off[sq];
      mine += nc > 1 ? nc - 1 : 0;
    }
    long long xs = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(kFull, xs, o);
      if (lane >= o) xs += y;
    }
    if (lane == 31) part[warp] = xs;
    __syncthreads();
    if (warp == 0) {
      long long ws = lane < kTableWarps ? part[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(kFull, ws, o);
        if (lane >= o) ws += y;
      }
      part[32 + lane] = ws;
    }
    __syncthreads();
    long long at = xs - mine + (warp > 0 ? part[32 + warp - 1] : 0);
    for (int64_t r = n0; r < n1; r++) {
      const int sq = seq_order[N - 1 - r];
      const long long nc = chunk_off[sq + 1] - chunk_off[sq];
      fill_off[sq] = (int32_t)at;
      at += nc > 1 ? nc - 1 : 0;
    }
    if (tid == 0) {
      hdr[kHdrFill1Chunks] = (int32_t)part[32 + kTableWarps - 1];
      // Equal chunk counts: every walk ends at about the same time, so the
      // fill waits for the walk grid once instead of checking its units.
      int uniform = 1;
      if (N > 0) {
        const int a = seq_order[0], b = seq_order[N - 1];
        uniform = chunk_off[a + 1] - chunk_off[a] == chunk_off[b + 1] - chunk_off[b];
      }
      hdr[kHdrFillUniform] = uniform;
    }
  }
  if (tid == 0) hdr[kHdrValid] = 1;
}

// ----------------------------------------------------------------------------
// Pass 1a: boundary prep of every full chunk (independent of the state)
// ----------------------------------------------------------------------------
// The prep kernel's AT shares memory with the key planes where they are big
// enough: the keys go to the pack once P = K K^T is formed.
template <int D, class IN>
constexpr bool prep_at_on_keys() {
  return Splits<IN>::K * kChunk * D * 2 >= (int)sizeof(PrepAT);
}
template <int D, class IN, bool ON_KEYS = prep_at_on_keys<D, IN>()>
struct PrepKernelSmem {
  PrepSmem<D, IN> prep;
  PrepAT AT;
  __device__ PrepAT& at() { return AT; }
};
template <int D, class IN>
struct PrepKernelSmem<D, IN, true> {
  PrepSmem<D, IN> prep;
  __device__ PrepAT& at() { return *reinterpret_cast<PrepAT*>(prep.K); }
};

template <int D, class IN>
__global__ void __launch_bounds__(kBndThreads, prep_at_on_keys<D, IN>() ? 4 : 3)
    k_prep(const IN* __restrict__ k, const IN* __restrict__ v, const float* __restrict__ beta,
           const float* __restrict__ g,
           const int32_t* __restrict__ cu, int H, const int32_t* __restrict__ hdr,
           const int32_t* __restrict__ chunk_off, const int32_t* __restrict__ chunk_seq,
           char* __restrict__ packs, int all_chunks, int n_seqs, int32_t* __restrict__ walk_done,
           const int32_t* __restrict__ fill_off, int32_t* __restrict__ fill_order) {
  static_assert(sizeof(PackHead<D, IN>) % 16 == 0 && sizeof(KVPlanes<D, IN>) % 16 == 0,
                "pack copies are 16-byte pieces");
  using PS = PrepSmem<D, IN>;
  using WP = WalkPack<D, IN>;
  static_assert(offsetof(PS, K) == sizeof(PackHead<D, IN>) &&
                    offsetof(WP, kv) == sizeof(PackHead<D, IN>),
                "head and key planes are contiguous in both layouts");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PrepKernelSmem<D, IN>& ks = *reinterpret_cast<PrepKernelSmem<D, IN>*>(smem_raw);
  PrepSmem<D, IN>& sm = ks.prep;
  const int c = blockIdx.x, h = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  if (hdr[kHdrValid] != 1) return;
  // The walk's word of unit (c, h) starts at zero; the fill order's entry of
  // chunk c (not a sequence's first) is written here.
  if (c < n_seqs && threadIdx.x == 0) walk_done[(size_t)c * H + h] = 0;
  if (c >= hdr[kHdrChunks]) return;
  const int n = chunk_seq[c];
  const int ci = c - chunk_off[n];
  if (h == 0 && ci >= 1 && threadIdx.x == 0) fill_order[fill_off[n] + ci - 1] = c;
  const int64_t L = (int64_t)cu[n + 1] - cu[n];
  // A trailing partial chunk has no boundary after it; with all_chunks (the
  // chunked forward's outputs need its pack) it is prepared zero-padded.
  const int rows = (int)min((int64_t)kChunk, L - (int64_t)ci * kChunk);
  if (rows < kChunk && !all_chunks) return;
  const int64_t t0 = (int64_t)cu[n] + (int64_t)ci * kChunk;
  const size_t tok = (size_t)t0 * H + h;
  // The tcgen05 walk copies the value planes from the inputs itself (a
  // tensor-map copy), so for it the pack carries the head and the keys; the
  // chunked layout's output kernel (all_chunks) reads the values from the pack.
  const bool vp = !use_tc<D, IN>() || all_chunks;
  PlaneRows<D, IN, kBndThreads> vrows;  // the chunk's values, in flight during the prep
  if (vp) vrows.load(v + tok * D, (size_t)H * D, rows);
  prep_stage<D, IN>(sm, k + tok * D, (size_t)H * D, beta + tok, g + tok, (size_t)H, rows);
  WalkPack<D, IN>& pk =
      *reinterpret_cast<WalkPack<D, IN>*>(packs + ((size_t)c * H + h) * pack_size<D, IN>());
  if constexpr (prep_at_on_keys<D, IN>()) {
    // Keys to the pack (bulk store) before AT overwrites them.
    bnd_prep<D, IN>(sm, ks.at(), [&]() {
      fence_async_smem();
      __syncthreads();
      if (threadIdx.x == 0) {
        bulk_store(pk.kv.K, smem_u32(sm.K), (uint32_t)sizeof(sm.K));
        bulk_commit();
        bulk_wait_read();
      }
      __syncthreads();
    });
  } else {
    bnd_prep<D, IN>(sm, ks.at());
  }
  // The head (and the keys, unless they are stored already) in one bulk
  // store: in shared memory they are contiguous, in the pack's layout.  The
  // value planes go from registers.
  constexpr uint32_t kOut =
      (uint32_t)(sizeof(PackHead<D, IN>) + (prep_at_on_keys<D, IN>() ? 0 : sizeof(sm.K)));
  fence_async_smem();
  __syncthreads();
  if (threadIdx.x == 0) {
    bulk_store(&pk.head, smem_u32(&sm.head), kOut);
    bulk_commit();
  }
  if (vp) vrows.store(pk.kv.V);
  if (threadIdx.x == 0) bulk_wait_read();  // shared memory must outlive the copy's reads
}

// ----------------------------------------------------------------------------
// Pass 1b: serial walk over the full chunks of one (sequence, head, row block)
// ----------------------------------------------------------------------------
// One block per (sequence, head): D/16 warps, 16 state rows each.
template <int D>
constexpr int walk_threads() { return 32 * (D / 16); }

template <int D, class IN>
struct WalkSmem {
  WalkPack<D, IN> buf[2];
  uint64_t ld_bar[2];
};

template <int D, class IN>
__global__ void __launch_bounds__(walk_threads<D>(), 1)
    k_walk(const int32_t* __restrict__ cu, int H, const float* __restrict__ h0,
           int32_t* __restrict__ hdr, const int32_t* __restrict__ chunk_off,
           const int32_t* __restrict__ seq_order, const char* __restrict__ packs,
           float* __restrict__ bstate,
           float* __restrict__ s_run_final, float* __restrict__ s_run_scale,
           float* __restrict__ s_bnd_final) {
  constexpr size_t PB = pack_size<D, IN>();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  WalkSmem<D, IN>& sm = *reinterpret_cast<WalkSmem<D, IN>*>(smem_raw);
  // One block per (sequence, head), sequences in the chunk table's order
  // (most chunks first).
  const int t = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (hdr[kHdrValid] != 1) return;
  const int n = seq_order[blockIdx.x / H], h = blockIdx.x % H;
  const int64_t L = (int64_t)cu[n + 1] - cu[n];
  const int64_t nf = L / kChunk, nc = (L + kChunk - 1) / kChunk;
  const int64_t base = chunk_off[n];
  const int r0 = 16 * (t >> 5);
  const size_t DD = (size_t)D * D;
  auto pack = [&](int64_t c) { return packs + ((size_t)(base + c) * H + h) * PB; };
  pack_bars_init(sm.ld_bar);
  float sacc[D / 8][4];
  if (h0) sacc_load<D>(sacc, h0 + ((size_t)n * H + h) * DD, r0);
  else sacc_zero<D>(sacc);
  if (nc > 0) sacc_store_bst<D>(sacc, bstate + ((size_t)base * H + h) * DD, r0);
  if (t == 0 && nf > 0) pack_fetch<D, IN>(sm.buf[0], pack(0), &sm.ld_bar[0]);
  int64_t issued = nf > 0 ? 1 : 0;
  bool ok = true;
  for (int64_t c = 0; c < nf; c++) {
    const size_t unit = (size_t)(base + c) * H + h;
    if (c + 1 < nf) {  // one chunk ahead into shared memory, two into L2
      if (t == 0) pack_fetch<D, IN>(sm.buf[(c + 1) & 1], pack(c + 1), &sm.ld_bar[(c + 1) & 1]);
      issued = c + 2;
    }
    if (c + 2 < nf && t == 0) prefetch_l2(pack(c + 2), (uint32_t)sizeof(WalkPack<D, IN>));
    if (__syncthreads_or(!pack_wait(sm.ld_bar, c))) {
      ok = false;
      pack_drain(sm.ld_bar, c, issued);
      break;
    }
    const WalkPack<D, IN>& b = sm.buf[c & 1];
    bnd_walk_warp<D, IN>(sacc, b.head, b.kv.K[0], b.kv.V[0], r0);
    if (c + 1 < nc) sacc_store_bst<D>(sacc, bstate + (unit + H) * DD, r0);
    __syncthreads();  // buffer c & 1 is refilled with chunk c + 2
  }
  if (!ok) {
    if (t == 0) atomicOr(&hdr[kHdrError], kErrTimeout);
    return;
  }
  const size_t so = ((size_t)n * H + h) * DD;
  if (s_bnd_final) sacc_store<D>(sacc, s_bnd_final + so, r0);
  if (s_run_final && (L % kChunk) == 0) {
    sacc_store<D>(sacc, s_run_final + so, r0);
    if (s_run_scale && t == 0) s_run_scale[(size_t)n * H + h] = 1.f;
  }
}

// The walk on tcgen05 (d = 128, bf16): one block of 256 threads per
// (sequence, head); warp w holds columns 64 (w / 4) .. + 63 of the rows of its
// tensor-memory lane quadrant (two column slices: 2.5 % faster per chunk step
// than four, and one slice spills registers; the bits do not depend on it).  Chunk c + 1's inputs are copied in (its pack
// head and key planes by one bulk copy, its value planes by one tensor-map
// copy from the input) from the start of chunk c's step, and chunk c + 2's
// pack prefetched into L2 while chunk c's products run.
// Each boundary state goes to the workspace through a shared-memory staging
// copy (permuted rows, conflict-free) and one bulk asynchronous store, issued
// with the chunk's first products.
constexpr int kWalkSlices = 2;
constexpr int kWalkThreads = kTcRows * kWalkSlices;

// Bytes of a walk pack ahead of its value planes (the head and the keys).
template <int D, class IN>
constexpr uint32_t pack_bytes_before_v() {
  using WP = WalkPack<D, IN>;
  return (uint32_t)offsetof(WP, kv.V);
}

// The fill's query, key and value maps; zeroed (never read) without tokens.
// A refused map is an error: there is no other route.
static cudaError_t row_maps(CUtensorMap* mq, CUtensorMap* mk, CUtensorMap* mv, const void* q,
                            const void* k, const void* v, int64_t T, int H) {
  memset(mq, 0, sizeof(*mq));
  memset(mk, 0, sizeof(*mk));
  memset(mv, 0, sizeof(*mv));
  if (T < 1) return cudaSuccess;
  const bool ok = encode_row_map(mq, q, T, H, 128, kChunk) &&
                  encode_row_map(mk, k, T, H, 128, kChunk) &&
                  encode_row_map(mv, v, T, H, 128, kChunk);
  return ok ? cudaSuccess : cudaErrorNotSupported;
}

// The tcgen05 walk's value map; zeroed (never read) when no sequence holds a
// full chunk.  A refused map is an error: there is no other route.
static cudaError_t value_map(CUtensorMap* mv, const void* v, int64_t T, int H) {
  memset(mv, 0, sizeof(*mv));
  if (T < kChunk) return cudaSuccess;
  return encode_plane_map(mv, v, T, H, 128, kChunk, 16) ? cudaSuccess : cudaErrorNotSupported;
}

// The tcgen05 walk's inputs of one full chunk into dst: the pack head and key
// planes by one bulk copy, the value planes by one tensor-map copy (tok0: the
// chunk's first token), all counted on the mbarrier at bar.  One thread.
template <int D, class IN>
__device__ __forceinline__ void pack_fetch_tc(WalkPack<D, IN>& dst, const char* pack,
                                              const CUtensorMap* mv, int tok0, int h,
                                              uint64_t* bar) {
  using WP = WalkPack<D, IN>;
  static_assert(sizeof(WP) % 128 == 0 && pack_bytes_before_v<D, IN>() % 128 == 0,
                "tensor-map destinations are 128-byte aligned");
  const uint32_t mb = smem_u32(bar);
  mbar_expect_tx(mb, (uint32_t)sizeof(WalkPack<D, IN>));
  bulk_load(smem_u32(&dst.head), pack, pack_bytes_before_v<D, IN>(), mb);
  tma_load_4d(smem_u32(dst.kv.V[0]), mv, 0, tok0, 0, h, mb);
}

template <int D, class IN>
struct WalkTcSmem {
  WalkPack<D, IN> buf[2];
  alignas(128) float stage[kTcRows * D];
  uint64_t ld_bar[2];
  uint64_t mbar;
  uint32_t tmem;
};

// Stage a thread's slice of the state (permuted rows) for a bulk store.
template <int D, int SC>
__device__ __forceinline__ void stage_slice(float* stage, const float* s, int row, int col0) {
  float* dst = stage + (size_t)row * D;
#pragma unroll
  for (int c = 0; c < SC; c += 4)
    *reinterpret_cast<float4*>(dst + bst_col(row, col0 + c)) =
        make_float4(s[c], s[c + 1], s[c + 2], s[c + 3]);
  fence_async_smem();
}

// The walk's work around the step of chunk c (warp-0 parts by lane 0):
// before the first barrier, issue chunk c + 1's copies into the buffer chunk
// c - 1 left (every thread is past its last read of it: the previous step
// ended with a block barrier), wait until the previous chunk's state store
// has read the staging buffer (thread 0) and for this chunk's inputs; issue
// chunk c + 2's L2 prefetch with the first products; stage the boundary
// state while they run and store it with the second round.
template <int D, class IN>
struct WalkHooks {
  WalkTcSmem<D, IN>* sm;
  int64_t c;
  const char* next;  // pack of chunk c + 1, or null
  const char* ahead; // pack of chunk c + 2, or null
  float* dst;        // boundary state of chunk c in the workspace
  int row, col0;
  const CUtensorMap* mv;  // value planes
  int tok_next, h;        // chunk c + 1's first token; the head
  __device__ bool inputs_ready() const {
    if (threadIdx.x == 0) {
      if (next) pack_fetch_tc<D, IN>(sm->buf[(c + 1) & 1], next, mv, tok_next, h,
                                     &sm->ld_bar[(c + 1) & 1]);
      bulk_wait_read();
    }
    return pack_wait(sm->ld_bar, c);
  }
  __device__ void after_first() const {
    if ((threadIdx.x & 31) != 0) return;
    if (ahead) prefetch_l2(ahead, pack_bytes_before_v<D, IN>());
  }
  __device__ void during_first(const float* s) const {
    stage_slice<D, D / kWalkSlices>(sm->stage, s, row, col0);
  }
  __device__ void after_second() const {
    if ((threadIdx.x & 31) != 0) return;
    bulk_store(dst, smem_u32(sm->stage), (uint32_t)(kTcRows * D * sizeof(float)));
    bulk_commit();
  }
  __device__ void after_last() const {}
};

template <int D, class IN>
__global__ void __launch_bounds__(kWalkThreads, 1)
    k_walk_tc(const int32_t* __restrict__ cu, int H, const float* __restrict__ h0,
              int32_t* __restrict__ hdr, const int32_t* __restrict__ chunk_off,
              const int32_t* __restrict__ seq_order, const char* __restrict__ packs,
              float* __restrict__ bstate,
              float* __restrict__ s_run_final, float* __restrict__ s_run_scale,
              float* __restrict__ s_bnd_final, int32_t* __restrict__ walk_done,
              const __grid_constant__ CUtensorMap map_v) {
  static_assert(use_tc<D, IN>(), "tcgen05 walk: d = 128, bf16 inputs");
  constexpr int SC = D / kWalkSlices;
  constexpr size_t PB = pack_size<D, IN>();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  WalkTcSmem<D, IN>& sm = *reinterpret_cast<WalkTcSmem<D, IN>*>(smem_raw);
  // One block per (sequence, head), sequences in the chunk table's order
  // (most chunks first).
  const int t = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (hdr[kHdrValid] != 1) return;
  const int n = seq_order[blockIdx.x / H], h = blockIdx.x % H;
  const int w = t >> 5, row = 32 * (w & 3) + (t & 31), col0 = SC * (w >> 2);
  const int64_t L = (int64_t)cu[n + 1] - cu[n];
  const int64_t nf = L / kChunk, nc = (L + kChunk - 1) / kChunk;
  const int64_t base = chunk_off[n];
  const size_t DD = (size_t)D * D;
  auto pack = [&](int64_t c) { return packs + ((size_t)(base + c) * H + h) * PB; };
  pack_bars_init(sm.ld_bar);
  TcCtx cx;
  tc_setup(cx, &sm.mbar, &sm.tmem);
  const int tok0 = cu[n];
  if (t == 0 && nf > 0)
    pack_fetch_tc<D, IN>(sm.buf[0], pack(0), &map_v, tok0, h, &sm.ld_bar[0]);
  if (t == 0 && nf > 1) prefetch_l2(pack(1), pack_bytes_before_v<D, IN>());
  float s[SC];
  if (h0) {
    const float* src = h0 + ((size_t)n * H + h) * DD + (size_t)row * D + col0;
#pragma unroll
    for (int c = 0; c < SC; c += 4) {
      const float4 x = *reinterpret_cast<const float4*>(src + c);
      s[c] = x.x;
      s[c + 1] = x.y;
      s[c + 2] = x.z;
      s[c + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < SC; i++) s[i] = 0.f;
  }
  int status = kStepDone;
  int64_t c = 0;
  for (; c < nf; c++) {
    const size_t unit = (size_t)(base + c) * H + h;
    const WalkHooks<D, IN> hooks{&sm, c, c + 1 < nf ? pack(c + 1) : nullptr,
                                 c + 2 < nf ? pack(c + 2) : nullptr, bstate + unit * DD, row,
                                 col0, &map_v, tok0 + (int)(c + 1) * kChunk, h};
    const WalkPack<D, IN>& b = sm.buf[c & 1];
    status = tc_walk_step<kWalkSlices>(s, b.head, b.kv.K[0], b.kv.V[0], cx, hooks);
    if (status != kStepDone) break;
  }
  if (status != kStepDone) {
    // Input copies possibly in flight: chunks c .. issued - 1 (the step issues
    // chunk c + 1's copies before its first barrier).
    const int64_t issued = c + 2 < nf ? c + 2 : nf;
    pack_drain(sm.ld_bar, c, issued);
    if (status == kStepFailed) tc_drain(cx);
    if (t == 0) atomicOr(&hdr[kHdrError], kErrTimeout);
  } else {
    if (nc > nf) {  // the trailing partial chunk starts from the last boundary
      if (t == 0) bulk_wait_read();
      __syncthreads();
      stage_slice<D, SC>(sm.stage, s, row, col0);
      __syncthreads();
      if (t == 0) {
        bulk_store(bstate + ((size_t)(base + nf) * H + h) * DD, smem_u32(sm.stage),
                   (uint32_t)(DD * sizeof(float)));
        bulk_commit();
      }
    }
    const size_t so = ((size_t)n * H + h) * DD + (size_t)row * D + col0;
#pragma unroll
    for (int i = 0; i < SC; i += 4) {
      const float4 x = make_float4(s[i], s[i + 1], s[i + 2], s[i + 3]);
      if (s_bnd_final) *reinterpret_cast<float4*>(s_bnd_final + so + i) = x;
      if (s_run_final && (L % kChunk) == 0) *reinterpret_cast<float4*>(s_run_final + so + i) = x;
    }
    if (s_run_final && s_run_scale && (L % kChunk) == 0 && t == 0)
      s_run_scale[(size_t)n * H + h] = 1.f;
  }
  if (t == 0) bulk_wait();  // every bulk store complete before the block exits
  if (status == kStepDone) {
    // Publish the unit: the block's stores (a barrier), then thread 0,
    // after its bulk stores completed, releases the unit's word, which the
    // fill acquires before it reads these states.
    __syncthreads();
    if (t == 0) {
      fence_proxy_async_global();
      __threadfence();
      st_release_gpu(&walk_done[(size_t)n * H + h], 1);
    }
  }
  tc_teardown(cx);
}

// ----------------------------------------------------------------------------
// Pass 2: per-token recurrence inside every chunk, from its boundary state.
// Persistent blocks (three per SM) take (chunk, head) items from a work
// counter.  An item's keys are widened to fp32 in shared memory (they are
// read twice per token); queries and values stay in the input dtype.  While
// an item runs, the next item's state and inputs are prefetched into L2.
// Which block runs an item does not change the item's bits.
// ----------------------------------------------------------------------------
template <int D, class IN, class OUT>
__global__ void __launch_bounds__(kFillThreads, 3)
    k_fill(const IN* __restrict__ q, const IN* __restrict__ k, const IN* __restrict__ v,
           const float* __restrict__ beta, const float* __restrict__ g,
           const int32_t* __restrict__ cu, int H, float scale, int32_t* __restrict__ hdr,
           const int32_t* __restrict__ chunk_off, const int32_t* __restrict__ chunk_seq,
           const float* __restrict__ bstate, OUT* __restrict__ o,
           float* __restrict__ s_run_final, float* __restrict__ s_run_scale, int n_seqs,
           const float* __restrict__ h0) {
  (void)n_seqs;
  (void)h0;
  constexpr int RT = D / 32, M4 = D / 16;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  FillSmem<D, IN>& sm = *reinterpret_cast<FillSmem<D, IN>*>(smem_raw);
  __shared__ int sh_item;
  pdl_wait();
  if (hdr[kHdrValid] != 1) return;
  const int n_items = hdr[kHdrChunks] * H;
  const int tid = threadIdx.x, l = tid & 3, r0 = (tid >> 2) * RT;
  const size_t DD = (size_t)D * D;

  if (tid == 0) sh_item = atomicAdd(&hdr[kHdrFillNext], 1);
  __syncthreads();
  int item = sh_item;
  while (item < n_items) {
    const FillItem cur = fill_item(item, H, cu, chunk_off, chunk_seq);
    fill_load<D, IN>(sm, cur, q, k, v, beta, g, H);
    Slice<RT, M4> S;
    slice_load_bst<RT, M4>(S, bstate + ((size_t)cur.c * H + cur.h) * DD, D, r0, l);
    if (tid == 0) sh_item = atomicAdd(&hdr[kHdrFillNext], 1);
    __syncthreads();
    const int next = sh_item;
    if (next < n_items)
      fill_prefetch<D, IN>(fill_item(next, H, cu, chunk_off, chunk_seq), bstate, q, k, v, H);

    float p[RT];
    slice_dot<RT, M4>(S, [&](int m) { return sld4(&sm.k[0][group_col(l, m)]); }, p);
#pragma unroll
    for (int i = 0; i < RT; i++) p[i] = quad_sum(p[i]);
    float c = 1.f;  // scale of the running state: 1 at the chunk boundary
    OUT* ob = o + ((size_t)cur.t0 * H + cur.h) * D + r0 + l;
    for (int t = 0; t < cur.len; t++) {
      float ov[RT];
      slice_token<true, RT, M4>(
          S, c, sm.a[t], sm.b[t], [&](int i) { return to_f(sm.v[t][r0 + i]); },
          [&](int m) { return sld4(&sm.k[t][group_col(l, m)]); },
          [&](int m) { return sld4(&sm.q[t][group_col(l, m)]); },
          [&](int m) { return sld4(&sm.k[t + 1][group_col(l, m)]); }, p, ov);
#pragma unroll
      for (int i = 0; i < RT; i++) ov[i] = __fmul_rn(scale, ov[i]);
      if (l < RT) st1(ob + (size_t)t * H * D, pick<RT>(ov, l));
    }
    const int64_t nc = (cur.L + kChunk - 1) / kChunk;
    if (s_run_final && cur.ci == nc - 1 && (cur.L % kChunk) != 0) {
      float* dst = s_run_final + ((size_t)cur.n * H + cur.h) * DD;
      if (s_run_scale) {
        slice_store<RT, M4>(S, dst, D, r0, l);
        if (tid == 0) s_run_scale[(size_t)cur.n * H + cur.h] = c;
      } else {
        slice_store_scaled<RT, M4>(S, c, dst, D, r0, l);
      }
    }
    item = next;
    __syncthreads();  // shared memory is reloaded for the next item
  }
}

// The two bf16 halves of a packed pair (the element at the lower address in
// the low half), exactly as fp32.
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }
constexpr int kFillWaitPolls = 1 << 22;

// ----------------------------------------------------------------------------
// Pass 2 at d = 128 with bf16 inputs: the same step, in the same order, with
// the quad reductions of gdn_fill.cuh (reduce-scatter of the row sums, the
// row's scalar work on its owning lane, all-gather of the update weight),
// keys and queries copied in by tensor map (while the item's state slice
// loads) and the keys widened to fp32 in shared memory once per item, the
// values copied in behind them, and the per-token scale sequence (c,
// c' = a c, 1 / c', renormalise) computed once per item (a left-to-right
// chain, then the reciprocals in parallel).  Bits are those of k_fill.
// ----------------------------------------------------------------------------
template <class OUT>
__global__ void __launch_bounds__(kFillThreads, 3)
    k_fill128(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
              const __nv_bfloat16* __restrict__ v, const float* __restrict__ beta,
              const float* __restrict__ g, const int32_t* __restrict__ cu, int H, float scale,
              int32_t* __restrict__ hdr, const int32_t* __restrict__ chunk_off,
              const int32_t* __restrict__ chunk_seq, const float* __restrict__ bstate,
              OUT* __restrict__ o, float* __restrict__ s_run_final,
              float* __restrict__ s_run_scale, int n_seqs, const float* __restrict__ h0,
              const int32_t* __restrict__ fill_order, const int32_t* walk_done,
              const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
              const __grid_constant__ CUtensorMap map_v) {
  constexpr int D = 128, M4 = D / 16;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Fill128Smem& sm = *reinterpret_cast<Fill128Smem*>(smem_raw);
  __shared__ int sh_item, sh_ready;
  // Two phases.  Phase 0: the first chunk of every sequence, whose entry
  // state is h0 (or zero), not a walk result, so that these items run on the
  // SMs the walk leaves idle (the walk only writes boundary states, the bound
  // final states and the pack reads, none of which a first chunk touches).
  // Phase 1: every other chunk, in the fill order (sequences with the fewest
  // chunks first: their walks end first).  An item starts once its unit's
  // walk word is set (acquired by thread 0, then a block barrier); the first
  // item whose word is not set yet makes the block wait for the whole walk
  // grid (griddepcontrol.wait), after which every word is.  The chunk table
  // (read in both phases) completed before the walk started.
  // A programmatic dependent (the backward's adjoint prep, which reads none of
  // this kernel's outputs) may start on the SMs this grid's tail leaves.
  pdl_trigger();
  if (hdr[kHdrValid] != 1) {
    pdl_wait();
    return;
  }
  const int tid = threadIdx.x, l = tid & 3, r0 = (tid >> 2) * 4, sg = quad_sigma(l);
  const int my_row = r0 + sg;
  const size_t DD = (size_t)D * D;

  for (int c = tid; c < D; c += kFillThreads) sm.k[kChunk][c] = 0.f;
  if (tid == 0) {
    mbar_init(smem_u32(&sm.bar[0]), 1);
    mbar_init(smem_u32(&sm.bar[1]), 1);
    fence_mbar_init();
  }
  uint32_t par = 0;     // phase of both barriers the next item waits for
  bool walked = false;  // this block has waited for the whole walk grid
  int phase = 0, limit = n_seqs * H;
  int32_t* counter = &hdr[kHdrFill0Next];
  auto claim = [&]() {
    __syncthreads();
    if (tid == 0) sh_item = atomicAdd(counter, 1);
    __syncthreads();
    return sh_item;
  };
  int item = claim();
  for (;;) {
    if (item >= limit) {
      if (phase == 1) break;
      phase = 1;
      counter = &hdr[kHdrFillNext];
      limit = hdr[kHdrFill1Chunks] * H;
      if (hdr[kHdrFillUniform]) {
        pdl_wait();  // the whole walk grid
        walked = true;
      }
      item = claim();
      continue;
    }
    FillItem cur;
    if (phase == 0) {
      const int n = item / H, hh = item - n * H;
      if (chunk_off[n] == chunk_off[n + 1]) {  // empty sequence
        item = claim();
        continue;
      }
      cur = fill_item(chunk_off[n] * H + hh, H, cu, chunk_off, chunk_seq);
    } else {
      cur = fill_item(fill_order[item / H] * H + item % H, H, cu, chunk_off, chunk_seq);
    }
    const size_t tb = (size_t)cur.t0 * H + cur.h;
    const uint32_t bar_kq = smem_u32(&sm.bar[0]), bar_v = smem_u32(&sm.bar[1]);
    // The item's keys (raw, into the value buffer) and queries by tensor-map
    // copies (rows past the item's length hold the next tokens or zeros and
    // are not read), while its scalars and the state slice load.
    if (tid == 0) {
      mbar_expect_tx(bar_kq, 2u * kChunk * D * 2);
      tma_load_3d(smem_u32(&sm.v[0][0]), &map_k, 0, cur.h, (int)cur.t0, bar_kq);
      tma_load_3d(smem_u32(&sm.q[0][0]), &map_q, 0, cur.h, (int)cur.t0, bar_kq);
    }
    // Per-token scalars: a = exp(g) and beta, two tokens per thread of warps
    // 0-1 in parallel.
    if (tid < kChunk) {
      float a = 0.f, b = 0.f;
      if (tid < cur.len) {
        a = step_decay(g[tb + (size_t)tid * H]);
        b = beta[tb + (size_t)tid * H];
      }
      sm.t0[tid] = make_float4(a, b, 0.f, 0.f);
    }
    // A phase-1 item's entry state is its unit's walk result: acquired here,
    // behind the input copies and scalar loads, which do not depend on it.
    if (phase == 1 && !walked) {
      if (tid == 0) sh_ready = ld_acquire_gpu(&walk_done[(size_t)cur.n * H + cur.h]);
      __syncthreads();
      if (!sh_ready) {
        pdl_wait();  // the whole walk grid
        walked = true;
      }
    }
    Slice<4, M4> S;
    if (phase == 0)
      slice4_load_plain<M4>(S, h0 ? h0 + ((size_t)cur.n * H + cur.h) * DD : nullptr, D, r0, sg,
                            l);
    else
      slice4_load_bst<M4>(S, bstate + ((size_t)cur.c * H + cur.h) * DD, D, r0, sg, l);
    // Keys widened to fp32; rows past the length are zero (row len is the
    // last token's next key).
    bool ok = mbar_wait(bar_kq, par, kFillWaitPolls);
    if (ok) {
#pragma unroll
      for (int j = 0; j < kChunk * D / 8 / kFillThreads; j++) {
        const int e = tid + j * kFillThreads, r = e >> 4, cc = (e & 15) * 8;
        const uint4 x = *reinterpret_cast<const uint4*>(&sm.v[r][cc]);
        float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
        if (r < cur.len) {
          lo = make_float4(bf_lo(x.x), bf_hi(x.x), bf_lo(x.y), bf_hi(x.y));
          hi = make_float4(bf_lo(x.z), bf_hi(x.z), bf_lo(x.w), bf_hi(x.w));
        }
        *reinterpret_cast<float4*>(&sm.k[r][cc]) = lo;
        *reinterpret_cast<float4*>(&sm.k[r][cc + 4]) = hi;
      }
    }
    if (__syncthreads_or(!ok)) {  // keys and queries never arrived: wait once more and stop
      if (tid == 0) atomicOr(&hdr[kHdrError], kErrTimeout);
      (void)mbar_wait(bar_kq, par, kFillWaitPolls);
      return;
    }
    // The raw keys are read: the values go to their buffer.
    if (tid == 0) {
      mbar_expect_tx(bar_v, (uint32_t)kChunk * D * 2);
      tma_load_3d(smem_u32(&sm.v[0][0]), &map_v, 0, cur.h, (int)cur.t0, bar_v);
    }
    // The scale sequence: a left-to-right chain that every lane of warp 0
    // follows (a_t read ahead from shared memory), keeping the values of its
    // own two tokens; then each lane writes its tokens' entries.
    if (tid < 32) {
      float c = 1.f, my_c[2] = {1.f, 1.f}, my_cn[2] = {0.f, 0.f};
      for (int t = 0; t < cur.len; t++) {
        const float cn = __fmul_rn(sm.t0[t].x, c);
        if (t == tid) { my_c[0] = c; my_cn[0] = cn; }
        if (t == tid + 32) { my_c[1] = c; my_cn[1] = cn; }
        c = scale_ok(cn) ? cn : 1.f;
      }
#pragma unroll
      for (int j = 0; j < 2; j++) {
        const int t = tid + 32 * j;
        if (t < cur.len) {
          const bool keep = scale_ok(my_cn[j]);
          sm.t0[t].z = my_c[j];
          sm.t0[t].w = keep ? my_cn[j] : 1.f;
          sm.t1[t] = make_float4(my_cn[j], keep ? __frcp_rn(my_cn[j]) : 0.f,
                                 keep ? 0.f : 1.f, 0.f);
        }
      }
    }
    float p_own;
    {
      float x[4];
      slice_dot<4, M4>(S, [&](int m) { return sld4(&sm.k[0][group_col(l, m)]); }, x);
      p_own = quad_rs(x);
    }
    ok = mbar_wait(bar_v, par, kFillWaitPolls);
    par ^= 1u;
    if (tid == 0) sh_item = atomicAdd(counter, 1);
    if (__syncthreads_or(!ok)) {  // the values never arrived: wait once more and stop
      if (tid == 0) atomicOr(&hdr[kHdrError], kErrTimeout);
      (void)mbar_wait(bar_v, par ^ 1u, kFillWaitPolls);
      return;
    }
    const int next = sh_item;
    if (phase == 1 && next < limit)
      fill_prefetch<D, __nv_bfloat16>(
          fill_item(fill_order[next / H] * H + next % H, H, cu, chunk_off, chunk_seq), bstate, q,
          k, v, H);

    float c = 1.f;  // scale of the running state: 1 at the chunk boundary
    OUT* ob = o + tb * D + my_row;
    for (int t = 0; t < cur.len; t++) {
      const float v_own = to_f(sm.v[t][my_row]);
      const float4 T0 = sm.t0[t], T1 = sm.t1[t];
      const float cn = T1.x, d = T1.y, cnew = T0.w;
      const bool keep = T1.z == 0.f;
      const float u = step_u(T0.x, T0.y, __fmul_rn(T0.z, p_own), v_own);
      auto fk = [&](int m) { return sld4(&sm.k[t][group_col(l, m)]); };
      auto fq = [&](int m) { return sld4(&sm.q[t][group_col(l, m)]); };
      auto fn = [&](int m) { return sld4(&sm.k[t + 1][group_col(l, m)]); };
      float w[4], oacc[4], pacc[4];
      if (keep) {
        quad_ag(__fmul_rn(u, d), w);
        slice_update<true, false, 4, M4>(S, cn, w, fk, fq, fn, oacc, pacc);
      } else {
        quad_ag(u, w);
        slice_update<true, true, 4, M4>(S, cn, w, fk, fq, fn, oacc, pacc);
      }
      c = cnew;
      p_own = quad_rs(pacc);
      st1(ob + (size_t)t * H * D, __fmul_rn(scale, __fmul_rn(cnew, quad_rs(oacc))));
    }
    const int64_t nc = (cur.L + kChunk - 1) / kChunk;
    if (s_run_final && cur.ci == nc - 1 && (cur.L % kChunk) != 0) {
      float* dst = s_run_final + ((size_t)cur.n * H + cur.h) * DD;
      if (s_run_scale) {
        slice4_store<M4>(S, dst, D, r0, sg, l);
        if (tid == 0) s_run_scale[(size_t)cur.n * H + cur.h] = c;
      } else {
        slice4_store_scaled<M4>(S, c, dst, D, r0, sg, l);
      }
    }
    item = next;
    __syncthreads();  // shared memory is reloaded for the next item
  }
  pdl_wait();  // the fill grid does not complete before the walk grid
}

// ----------------------------------------------------------------------------
// Chunk boundary over a buffer: decode resync (RESYNC) or gdn_chunk_boundary
// ----------------------------------------------------------------------------
template <int D, class IN>
struct BndSmem {
  PrepSmem<D, IN> prep;
  PrepAT AT;
  alignas(16) __nv_bfloat16 V[Splits<IN>::K][kChunk * D];
};

// The tcgen05 form keeps the walk's operands in tensor memory.
template <int D, class IN>
struct BndTcSmem {
  PrepSmem<D, IN> prep;
  PrepAT AT;
  alignas(16) __nv_bfloat16 V[Splits<IN>::K][kChunk * D];
  uint64_t mbar;
  uint32_t tmem;
};

template <int D, class IN>
using BndUnitSmem = typename std::conditional<use_tc<D, IN>(), BndTcSmem<D, IN>, BndSmem<D, IN>>::type;

// Threads of a block that runs whole chunk boundaries: the tcgen05 walk uses
// kWalkSlices column slices (256 threads), the mma.sync walk 128 threads.
template <int D, class IN>
constexpr int unit_threads() {
  return use_tc<D, IN>() ? kTcRows * kWalkSlices : kBndThreads;
}

// One chunk boundary for `unit` (prep + walk of all D rows), in place allowed,
// by a block of unit_threads<D, IN>() threads.  Returns false if a
// tensor-core wait gave up (the unit's s_end is then NaN).
template <int D, class IN>
__device__ __forceinline__ bool bnd_unit(BndUnitSmem<D, IN>& sm, const float* s_start,
                                         const IN* kb, const IN* vb, const float* bb,
                                         const float* gb, size_t unit, float* s_end) {
  constexpr int NT = unit_threads<D, IN>();
  const size_t DD = (size_t)D * D;
  stage_planes<D, IN>(sm.V, vb + unit * kChunk * D, (size_t)D, NT);
  prep_stage<D, IN>(sm.prep, kb + unit * kChunk * D, (size_t)D, bb + unit * kChunk,
                    gb + unit * kChunk, 1);
  if constexpr (use_tc<D, IN>()) {
    constexpr int SC = D / kWalkSlices;
    // The state's loads are issued before the prep, which does not need them.
    const int w = threadIdx.x >> 5, row = 32 * (w & 3) + (threadIdx.x & 31);
    const size_t off = unit * DD + (size_t)row * D + SC * (w >> 2);
    float s[SC];
#pragma unroll
    for (int c = 0; c < SC; c += 4) {
      const float4 x = *reinterpret_cast<const float4*>(s_start + off + c);
      s[c] = x.x;
      s[c + 1] = x.y;
      s[c + 2] = x.z;
      s[c + 3] = x.w;
    }
    bnd_prep<D, IN>(sm.prep, sm.AT);
    TcCtx cx;
    tc_setup(cx, &sm.mbar, &sm.tmem);
    const int st =
        tc_walk_step<kWalkSlices>(s, sm.prep.head, sm.prep.K[0], sm.V[0], cx, TcNoHooks{});
    if (st != kStepDone) {
      if (st == kStepFailed) tc_drain(cx);
#pragma unroll
      for (int i = 0; i < SC; i++) s[i] = __int_as_float(0x7fc00000);
    }
#pragma unroll
    for (int c = 0; c < SC; c += 4)
      *reinterpret_cast<float4*>(s_end + off + c) = make_float4(s[c], s[c + 1], s[c + 2], s[c + 3]);
    tc_teardown(cx);
    __syncthreads();  // shared memory is reused by the next unit
    return st == kStepDone;
  } else {
    bnd_prep<D, IN>(sm.prep, sm.AT);
    const int warp = threadIdx.x >> 5;
#pragma unroll 1
    for (int rt = 0; rt < D / 64; rt++) {
      const int r0 = 16 * warp + 64 * rt;
      float sacc[D / 8][4];
      sacc_load<D>(sacc, s_start + unit * DD, r0);
      bnd_walk_warp<D, IN>(sacc, sm.prep.head, sm.prep.K[0], sm.V[0], r0);
      sacc_store<D>(sacc, s_end + unit * DD, r0);
    }
    __syncthreads();  // shared memory is reused by the next unit
    return true;
  }
}

// gdn_chunk_boundary: one block per (row, head).
template <int D, class IN>
__global__ void __launch_bounds__(unit_threads<D, IN>())
    k_bnd(const float* s_start, const IN* __restrict__ kb, const IN* __restrict__ vb,
          const float* __restrict__ bb, const float* __restrict__ gb, int H, float* s_end) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  BndUnitSmem<D, IN>& sm = *reinterpret_cast<BndUnitSmem<D, IN>*>(smem_raw);
  bnd_unit<D, IN>(sm, s_start, kb, vb, bb, gb, (size_t)blockIdx.x * H + blockIdx.y, s_end);
}

// ----------------------------------------------------------------------------
// Decode step: one block per (row, head) unit.  The block that appends the
// last token of a chunk then runs the chunk boundary for its unit (the
// resync), while the other units' blocks are still stepping.
// ----------------------------------------------------------------------------
constexpr int kDecThreads = 128;  // four state rows per thread

// Words of a decode state's resync work list.
constexpr int kResyncCount = 0;  // units listed by this step
constexpr int kResyncNext = 1;   // work counter of k_resync
constexpr int kResyncDone = 2;   // k_resync blocks finished
constexpr int kResyncList = 4;   // the units

template <int D, class IN, class OUT>
__global__ void __launch_bounds__(kDecThreads)
    k_dec_step(const IN* __restrict__ q, const IN* __restrict__ k, const IN* __restrict__ v,
               const float* __restrict__ beta, const float* __restrict__ g,
               const int32_t* __restrict__ slot_idx, int H, float scale, float* s_run,
               float* s_scale, float* s_bnd, IN* buf_k, IN* buf_v, float* buf_beta,
               float* buf_g, int32_t* pos, int32_t* error, int32_t* resync, int n_slots,
               OUT* __restrict__ o) {
  constexpr int RT = D / 32, M4 = D / 16;
  __shared__ int sh_pos, sh_slot;
  pdl_trigger();  // the resync may be scheduled; it waits for this grid
  const int b = blockIdx.x, h = blockIdx.y;
  const int tid = threadIdx.x, l = tid & 3, r0 = (tid >> 2) * RT;
  if (tid == 0) {
    const int slot = slot_idx ? slot_idx[b] : b;
    int p0 = -1;
    if (slot >= 0 && slot < n_slots) p0 = pos[(size_t)slot * H + h];
    if (p0 < 0 || p0 >= kChunk) {
      atomicOr(error, kErrPos);
      p0 = -1;
    }
    sh_pos = p0;
    sh_slot = slot;
  }
  __syncthreads();
  const int p0 = sh_pos;
  if (p0 < 0) return;
  const size_t unit = (size_t)sh_slot * H + h;
  const size_t DD = (size_t)D * D;
  const size_t tok = (size_t)b * H + h;
  Slice<RT, M4> S;
  slice_load<RT, M4>(S, (p0 == 0 ? s_bnd : s_run) + unit * DD, D, r0, l);
  const IN* kp = k + tok * D;
  const IN* qp = q + tok * D;
  const float a = step_decay(g[tok]);
  const float bt = beta[tok];
  float c = (p0 == 0) ? 1.f : s_scale[unit];
  float p[RT], ov[RT];
  auto kf = [&](int m) { return ld4(kp + group_col(l, m)); };
  slice_dot<RT, M4>(S, kf, p);
#pragma unroll
  for (int i = 0; i < RT; i++) p[i] = quad_sum(p[i]);
  slice_token<false, RT, M4>(
      S, c, a, bt, [&](int i) { return ld1(v + tok * D + r0 + i); }, kf,
      [&](int m) { return ld4(qp + group_col(l, m)); },
      [&](int m) { return make_float4(0.f, 0.f, 0.f, 0.f); }, p, ov);
#pragma unroll
  for (int i = 0; i < RT; i++) ov[i] = __fmul_rn(scale, ov[i]);
  if (l < RT) st1(o + tok * D + r0 + l, pick<RT>(ov, l));
  if (p0 + 1 < kChunk) {
    slice_store<RT, M4>(S, s_run + unit * DD, D, r0, l);
    if (tid == 0) s_scale[unit] = c;
  }
  // append the token to the chunk buffer (bit copies)
  const size_t brow = (unit * kChunk + p0) * D;
  for (int e = tid; e < D; e += kDecThreads) {
    buf_k[brow + e] = k[tok * D + e];
    buf_v[brow + e] = v[tok * D + e];
  }
  if (tid == 0) {
    buf_beta[unit * kChunk + p0] = bt;
    buf_g[unit * kChunk + p0] = g[tok];
    if (p0 + 1 < kChunk) pos[unit] = p0 + 1;
  }
  if (p0 + 1 == kChunk && tid == 0) {
    // The buffer is full: k_resync advances the boundary state over its C
    // tokens, and that becomes the running state of the next step (pos = 0).
    const int j = atomicAdd(&resync[kResyncCount], 1);
    if (j < n_slots * H) resync[kResyncList + j] = (int32_t)unit;
    else atomicOr(error, kErrPos);  // rows naming the same slot twice
    pos[unit] = 0;
  }
}

// The chunk boundary of every unit that k_dec_step listed, in place on s_bnd.
// Persistent blocks take list entries from a counter; the last block to
// finish empties the list for the next step.
template <int D, class IN>
__global__ void __launch_bounds__(unit_threads<D, IN>())
    k_resync(int H, float* s_bnd, const IN* buf_k, const IN* buf_v, const float* buf_beta,
             const float* buf_g, int32_t* resync, int n_slots, int32_t* error) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  BndUnitSmem<D, IN>& sm = *reinterpret_cast<BndUnitSmem<D, IN>*>(smem_raw);
  __shared__ int sh_j;
  pdl_wait();  // the step kernel's list and buffers
  const int count = min(resync[kResyncCount], n_slots * H);
  for (;;) {
    if (threadIdx.x == 0) sh_j = atomicAdd(&resync[kResyncNext], 1);
    __syncthreads();
    const int j = sh_j;
    __syncthreads();  // every thread has j before thread 0 takes the next one
    if (j >= count) break;
    const size_t unit = (size_t)resync[kResyncList + j];
    if (!bnd_unit<D, IN>(sm, s_bnd, buf_k, buf_v, buf_beta, buf_g, unit, s_bnd) &&
        threadIdx.x == 0)
      atomicOr(error, kErrTimeout);
  }
  if (threadIdx.x == 0 && atomicAdd(&resync[kResyncDone], 1) == (int)gridDim.x - 1) {
    resync[kResyncCount] = 0;  // every block has read the count and left the loop
    resync[kResyncNext] = 0;
    resync[kResyncDone] = 0;
  }
}

// ----------------------------------------------------------------------------
// Prefill -> decode handoff
// ----------------------------------------------------------------------------
template <int D, class IN>
__global__ void __launch_bounds__(128)
    k_handoff(const IN* __restrict__ k, const IN* __restrict__ v, const float* __restrict__ beta,
              const float* __restrict__ g, const int32_t* __restrict__ cu, int64_t T, int H,
              const float* __restrict__ s_run_final, const float* __restrict__ s_run_scale,
              const float* __restrict__ s_bnd_final, const int32_t* __restrict__ slot_idx,
              float* s_run, float* s_scale, float* s_bnd, IN* buf_k,
              IN* buf_v, float* buf_beta, float* buf_g, int32_t* pos, int32_t* error,
              int n_slots) {
  const int n = blockIdx.x, h = blockIdx.y;
  const int slot = slot_idx ? slot_idx[n] : n;
  const int64_t c0 = cu[n], c1 = cu[n + 1];
  if (slot < 0 || slot >= n_slots || c0 < 0 || c1 < c0 || c1 > T) {
    if (threadIdx.x == 0) atomicOr(error, slot < 0 || slot >= n_slots ? kErrPos : kErrCuSeqlens);
    return;
  }
  const int rem = (int)((c1 - c0) % kChunk);
  const size_t unit = (size_t)slot * H + h, src = (size_t)n * H + h;
  const size_t DD = (size_t)D * D;
  for (size_t e = threadIdx.x; e < DD / 4; e += 128) {
    reinterpret_cast<float4*>(s_run + unit * DD)[e] =
        reinterpret_cast<const float4*>(s_run_final + src * DD)[e];
    reinterpret_cast<float4*>(s_bnd + unit * DD)[e] =
        reinterpret_cast<const float4*>(s_bnd_final + src * DD)[e];
  }
  for (int e = threadIdx.x; e < rem * D; e += 128) {
    const int i = e / D, c = e % D;
    const size_t t = (size_t)(c1 - rem + i);
    buf_k[(unit * kChunk + i) * D + c] = k[(t * H + h) * D + c];
    buf_v[(unit * kChunk + i) * D + c] = v[(t * H + h) * D + c];
  }
  for (int i = threadIdx.x; i < rem; i += 128) {
    const size_t t = (size_t)(c1 - rem + i);
    buf_beta[unit * kChunk + i] = beta[t * H + h];
    buf_g[unit * kChunk + i] = g[t * H + h];
  }
  if (threadIdx.x == 0) {
    pos[unit] = rem;
    s_scale[unit] = s_run_scale ? s_run_scale[src] : 1.f;
  }
}

// ----------------------------------------------------------------------------
// Host launchers
// ----------------------------------------------------------------------------
template <class KernelT>
static cudaError_t set_smem(KernelT kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

#define GDN_TRY(expr)                 \
  do {                                \
    cudaError_t e_ = (expr);          \
    if (e_ != cudaSuccess) return e_; \
  } while (0)

// Persistent grid size of a kernel: resident blocks per SM x SMs.
template <class KernelT>
static cudaError_t persistent_grid(KernelT kern, int threads, size_t smem, int* grid) {
  int dev = 0, sms = 0, per_sm = 0;
  GDN_TRY(cudaGetDevice(&dev));
  GDN_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  GDN_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem));
  *grid = (per_sm > 0 ? per_sm : 1) * sms;
  return cudaSuccess;
}

// The fill kernel of a (d, dtype): k_fill128 at d = 128 with bf16 inputs,
// k_fill otherwise.  Both take the same arguments and give the same bits.
template <int D, class IN, class OUT>
static auto fill_kernel() {
  if constexpr (D == 128 && sizeof(IN) == 2)
    return k_fill128<OUT>;
  else
    return k_fill<D, IN, OUT>;
}
template <int D, class IN>
static constexpr size_t fill_smem() {
  if constexpr (D == 128 && sizeof(IN) == 2)
    return sizeof(Fill128Smem);
  else
    return sizeof(FillSmem<D, IN>);
}

template <int D, class IN, class OUT>
static cudaError_t forward_impl(const FwdArgs& a, cudaStream_t st) {
  static_assert(pack_size<D, IN>() == pack_bytes(D, sizeof(IN) == 2), "pack layout mismatch");
  const FwdLayout& L = a.lay;
  char* ws = a.ws;
  int32_t* hdr = reinterpret_cast<int32_t*>(ws + L.hdr);
  int32_t* chunk_off = reinterpret_cast<int32_t*>(ws + L.chunk_off);
  int32_t* chunk_seq = reinterpret_cast<int32_t*>(ws + L.chunk_seq);
  float* bstate = reinterpret_cast<float*>(ws + L.bstate);
  char* packs = ws + L.pack;
  const IN* q = static_cast<const IN*>(a.q);
  const IN* k = static_cast<const IN*>(a.k);
  const IN* v = static_cast<const IN*>(a.v);
  auto mark = [&](int i) -> cudaError_t {
    return a.events ? cudaEventRecord(static_cast<cudaEvent_t>(a.events[i]), st) : cudaSuccess;
  };
  GDN_TRY(mark(0));
  int32_t* seq_order = reinterpret_cast<int32_t*>(ws + L.seq_order);
  int32_t* walk_done = reinterpret_cast<int32_t*>(ws + L.walk_done);
  int32_t* fill_off = reinterpret_cast<int32_t*>(ws + L.fill_off);
  int32_t* fill_order = reinterpret_cast<int32_t*>(ws + L.fill_order);
  k_chunk_table<<<1, kTableThreads, 0, st>>>(a.cu_seqlens, a.n_seqs, a.T, a.H, hdr, chunk_off,
                                             seq_order, chunk_seq, fill_off, L.max_chunks);
  GDN_TRY(cudaGetLastError());
  const dim3 gchunks((unsigned)L.max_chunks, (unsigned)a.H);
  GDN_TRY(mark(1));
  {
    // prep, walk and fill are programmatic dependents of the kernel before
    // them (each waits for it in pdl_wait before touching memory)
    auto kern = k_prep<D, IN>;
    const size_t sm = sizeof(PrepKernelSmem<D, IN>);
    GDN_TRY(set_smem(kern, sm));
    GDN_TRY(launch_dependent(kern, gchunks, dim3(kBndThreads), sm, st, k, v, a.beta, a.g,
                             a.cu_seqlens, a.H, (const int32_t*)hdr, (const int32_t*)chunk_off,
                             (const int32_t*)chunk_seq, packs, 0, a.n_seqs, walk_done,
                             (const int32_t*)fill_off, fill_order));
  }
  GDN_TRY(mark(2));
  const dim3 gunits((unsigned)((size_t)a.n_seqs * a.H));
  if constexpr (use_tc<D, IN>()) {
    auto kern = k_walk_tc<D, IN>;
    const size_t sm = sizeof(WalkTcSmem<D, IN>);
    GDN_TRY(set_smem(kern, sm));
    CUtensorMap mv;
    GDN_TRY(value_map(&mv, v, a.T, a.H));
    GDN_TRY(launch_dependent(kern, gunits, dim3(kWalkThreads), sm, st, a.cu_seqlens, a.H, a.h0,
                             hdr, (const int32_t*)chunk_off, (const int32_t*)seq_order,
                             (const char*)packs, bstate, a.s_run_final, a.s_run_scale,
                             a.s_bnd_final, walk_done, mv));
  } else {
    auto kern = k_walk<D, IN>;
    const size_t sm = sizeof(WalkSmem<D, IN>);
    GDN_TRY(set_smem(kern, sm));
    GDN_TRY(launch_dependent(kern, gunits, dim3(walk_threads<D>()), sm, st, a.cu_seqlens, a.H,
                             a.h0, hdr, (const int32_t*)chunk_off, (const int32_t*)seq_order,
                             (const char*)packs, bstate, a.s_run_final, a.s_run_scale,
                             a.s_bnd_final));
  }
  GDN_TRY(mark(3));
  if (!a.pass1_only) {
    auto kern = fill_kernel<D, IN, OUT>();
    const size_t sm = fill_smem<D, IN>();
    GDN_TRY(set_smem(kern, sm));
    int grid = 0;
    GDN_TRY(persistent_grid(kern, kFillThreads, sm, &grid));
    const int64_t items = L.max_chunks * a.H;
    if ((int64_t)grid > items) grid = (int)items;
    if constexpr (D == 128 && sizeof(IN) == 2) {
      CUtensorMap mq, mk, mv;
      GDN_TRY(row_maps(&mq, &mk, &mv, q, k, v, a.T, a.H));
      GDN_TRY(launch_dependent(kern, dim3((unsigned)grid), dim3(kFillThreads), sm, st, q, k, v,
                               a.beta, a.g, a.cu_seqlens, a.H, a.scale, hdr,
                               (const int32_t*)chunk_off, (const int32_t*)chunk_seq,
                               (const float*)bstate, static_cast<OUT*>(a.o), a.s_run_final,
                               a.s_run_scale, a.n_seqs, a.h0, (const int32_t*)fill_order,
                               (const int32_t*)walk_done, mq, mk, mv));
    } else {
      GDN_TRY(launch_dependent(kern, dim3((unsigned)grid), dim3(kFillThreads), sm, st, q, k, v,
                               a.beta, a.g, a.cu_seqlens, a.H, a.scale, hdr,
                               (const int32_t*)chunk_off, (const int32_t*)chunk_seq,
                               (const float*)bstate, static_cast<OUT*>(a.o), a.s_run_final,
                               a.s_run_scale, a.n_seqs, a.h0));
    }
  }
  return mark(4);
}

// The chunked ("native mixed") forward, d = 128 with bf16 inputs: the CPR
// first pass with every chunk prepared (trailing partial chunks zero-padded),
// then the output products of gdn_native.cuh from the chunks' entry states.
template <class OUT>
static cudaError_t native_impl(const FwdArgs& a, cudaStream_t st) {
  using IN = __nv_bfloat16;
  constexpr int D = 128;
  const FwdLayout& L = a.lay;
  char* ws = a.ws;
  int32_t* hdr = reinterpret_cast<int32_t*>(ws + L.hdr);
  int32_t* chunk_off = reinterpret_cast<int32_t*>(ws + L.chunk_off);
  int32_t* chunk_seq = reinterpret_cast<int32_t*>(ws + L.chunk_seq);
  float* bstate = reinterpret_cast<float*>(ws + L.bstate);
  char* packs = ws + L.pack;
  auto mark = [&](int i) -> cudaError_t {
    return a.events ? cudaEventRecord(static_cast<cudaEvent_t>(a.events[i]), st) : cudaSuccess;
  };
  GDN_TRY(mark(0));
  int32_t* seq_order = reinterpret_cast<int32_t*>(ws + L.seq_order);
  int32_t* walk_done = reinterpret_cast<int32_t*>(ws + L.walk_done);
  int32_t* fill_off = reinterpret_cast<int32_t*>(ws + L.fill_off);
  int32_t* fill_order = reinterpret_cast<int32_t*>(ws + L.fill_order);
  k_chunk_table<<<1, kTableThreads, 0, st>>>(a.cu_seqlens, a.n_seqs, a.T, a.H, hdr, chunk_off,
                                             seq_order, chunk_seq, fill_off, L.max_chunks);
  GDN_TRY(cudaGetLastError());
  GDN_TRY(mark(1));
  {
    auto kern = k_prep<D, IN>;
    const size_t sm = sizeof(PrepKernelSmem<D, IN>);
    GDN_TRY(set_smem(kern, sm));
    kern<<<dim3((unsigned)L.max_chunks, (unsigned)a.H), kBndThreads, sm, st>>>(
        static_cast<const IN*>(a.k), static_cast<const IN*>(a.v), a.beta, a.g, a.cu_seqlens,
        a.H, hdr, chunk_off, chunk_seq, packs, 1, a.n_seqs, walk_done, fill_off, fill_order);
    GDN_TRY(cudaGetLastError());
  }
  GDN_TRY(mark(2));
  {
    auto kern = k_walk_tc<D, IN>;
    const size_t sm = sizeof(WalkTcSmem<D, IN>);
    GDN_TRY(set_smem(kern, sm));
    CUtensorMap mv;
    GDN_TRY(value_map(&mv, a.v, a.T, a.H));
    kern<<<(unsigned)((size_t)a.n_seqs * a.H), kWalkThreads, sm, st>>>(
        a.cu_seqlens, a.H, a.h0, hdr, chunk_off, seq_order, packs, bstate, a.s_run_final, nullptr,
        a.s_bnd_final, walk_done, mv);
    GDN_TRY(cudaGetLastError());
  }
  GDN_TRY(mark(3));
  {
    auto kern = k_native_tc<OUT>;
    const size_t sm = sizeof(NativeSmem);
    GDN_TRY(set_smem(kern, sm));
    int dev = 0, sms = 0;
    GDN_TRY(cudaGetDevice(&dev));
    GDN_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const int64_t items = L.max_chunks * a.H;
    const int grid = (int)(items < sms ? items : sms);
    kern<<<grid, kNtThreads, sm, st>>>(static_cast<const IN*>(a.q), a.g, a.cu_seqlens, a.H,
                                       a.scale, hdr, chunk_off, chunk_seq, packs, bstate,
                                       static_cast<OUT*>(a.o), a.s_run_final);
    GDN_TRY(cudaGetLastError());
  }
  return mark(4);
}

template <int D, class IN, class OUT>
static cudaError_t decode_impl(const DecArgs& a, cudaStream_t st) {
  k_dec_step<D, IN, OUT><<<dim3((unsigned)a.B, (unsigned)a.H), kDecThreads, 0, st>>>(
      static_cast<const IN*>(a.q), static_cast<const IN*>(a.k), static_cast<const IN*>(a.v),
      a.beta, a.g, a.slot_idx, a.H, a.scale, a.s_run, a.s_scale, a.s_bnd,
      static_cast<IN*>(a.buf_k), static_cast<IN*>(a.buf_v), a.buf_beta, a.buf_g, a.pos, a.error,
      a.resync, a.n_slots, static_cast<OUT*>(a.o));
  GDN_TRY(cudaGetLastError());
  auto kern = k_resync<D, IN>;
  const size_t sm = sizeof(BndUnitSmem<D, IN>);
  GDN_TRY(set_smem(kern, sm));
  int grid = 0;
  GDN_TRY(persistent_grid(kern, unit_threads<D, IN>(), sm, &grid));
  return launch_dependent(kern, dim3((unsigned)grid), dim3(unit_threads<D, IN>()), sm, st, a.H,
                          a.s_bnd, static_cast<const IN*>(a.buf_k),
                          static_cast<const IN*>(a.buf_v), (const float*)a.buf_beta,
                          (const float*)a.buf_g, a.resync, a.n_slots, a.error);
}

template <int D, class IN>
static cudaError_t handoff_impl(const HandoffArgs& a, cudaStream_t st) {
  k_handoff<D, IN><<<dim3((unsigned)a.n_seqs, (unsigned)a.H), 128, 0, st>>>(
      static_cast<const IN*>(a.k), static_cast<const IN*>(a.v), a.beta, a.g, a.cu_seqlens, a.T,
      a.H, a.s_run_final, a.s_run_scale, a.s_bnd_final, a.slot_idx, a.s_run, a.s_scale, a.s_bnd,
      static_cast<IN*>(a.buf_k), static_cast<IN*>(a.buf_v), a.buf_beta, a.buf_g, a.pos,
      a.error, a.n_slots);
  return cudaGetLastError();
}

template <int D, class IN>
static cudaError_t boundary_impl(const BndArgs& a, cudaStream_t st) {
  auto kern = k_bnd<D, IN>;
  const size_t sm = sizeof(BndUnitSmem<D, IN>);
  GDN_TRY(set_smem(kern, sm));
  kern<<<dim3((unsigned)a.B, (unsigned)a.H), unit_threads<D, IN>(), sm, st>>>(
      a.s_start, static_cast<const IN*>(a.k), static_cast<const IN*>(a.v), a.beta, a.g, a.H,
      a.s_end);
  return cudaGetLastError();
}

using bf16 = __nv_bfloat16;

cudaError_t launch_forward(const FwdArgs& a, cudaStream_t st) {
  if (a.D == 64) {
    if (a.in_bf16)
      return a.out_bf16 ? forward_impl<64, bf16, bf16>(a, st) : forward_impl<64, bf16, float>(a, st);
    return a.out_bf16 ? forward_impl<64, float, bf16>(a, st) : forward_impl<64, float, float>(a, st);
  }
  if (!a.in_bf16) return cudaErrorNotSupported;  // fp32 inputs: d = 64 only
  return a.out_bf16 ? forward_impl<128, bf16, bf16>(a, st) : forward_impl<128, bf16, float>(a, st);
}

cudaError_t launch_native_forward(const FwdArgs& a, cudaStream_t st) {
  if (a.D != 128 || !a.in_bf16) return cudaErrorNotSupported;
  return a.out_bf16 ? native_impl<bf16>(a, st) : native_impl<float>(a, st);
}

cudaError_t launch_decode_step(const DecArgs& a, cudaStream_t st) {
  if (a.D == 64) {
    if (a.in_bf16)
      return a.out_bf16 ? decode_impl<64, bf16, bf16>(a, st) : decode_impl<64, bf16, float>(a, st);
    return a.out_bf16 ? decode_impl<64, float, bf16>(a, st) : decode_impl<64, float, float>(a, st);
  }
  if (!a.in_bf16) return cudaErrorNotSupported;  // fp32 inputs: d = 64 only
  return a.out_bf16 ? decode_impl<128, bf16, bf16>(a, st) : decode_impl<128, bf16, float>(a, st);
}

cudaError_t launch_handoff(const HandoffArgs& a, cudaStream_t st) {
  if (a.D == 64) return a.in_bf16 ? handoff_impl<64, bf16>(a, st) : handoff_impl<64, float>(a, st);
  if (!a.in_bf16) return cudaErrorNotSupported;  // fp32 inputs: d = 64 only
  return handoff_impl<128, bf16>(a, st);
}

cudaError_t launch_chunk_boundary(const BndArgs& a, cudaStream_t st) {
  if (a.D == 64) return a.in_bf16 ? boundary_impl<64, bf16>(a, st) : boundary_impl<64, float>(a, st);
  if (!a.in_bf16) return cudaErrorNotSupported;  // fp32 inputs: d = 64 only
  return boundary_impl<128, bf16>(a, st);
}

}  // namespace gdn
