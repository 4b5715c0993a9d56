/*
 * gdn_cpr.h -- C ABI of the CPR Gated DeltaNet library (libgdn_cpr.so).
 *
 * The layer: "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI
 * Training Runs", section "Solving the linear-attention headache".  Gated
 * DeltaNet is evaluated by CPR (chunkwise-parallel recurrent).  The token
 * recurrence is what gets computed; the chunks only organise the work.  A
 * serial sweep over chunk starts produces the state that enters each chunk;
 * then every chunk replays the token recurrence from its entry state, all
 * chunks at once.  Decode steps the same recurrence one token at a time and,
 * whenever a chunk's worth of tokens has gone by, replaces its state by the
 * one the chunk-start computation gives.  Training, prefill and decode thus
 * round identically.  The recurrence (one state per sequence and head):
 *
 *     S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t,        alpha_t = exp(g_t)
 *
 * S is d_v x d_k, stored row-major (row = value channel, contiguous over the
 * key channel), fp32.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every data pointer is caller-owned DEVICE memory on the current device.
 *   The library allocates no device memory; scratch space is the caller's
 *   `workspace`.  Pointers must be 16-byte aligned.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  All calls are asynchronous on it and never synchronise the
 *   host, except gdn_check_error.
 * - Argument errors are detected on the host before anything is launched
 *   and returned synchronously (GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED,
 *   GDN_ERR_WORKSPACE).  A failed launch returns GDN_ERR_CUDA.  Bad device
 *   data (for example a decreasing cu_seqlens) cannot be seen on the host:
 *   the kernels skip the affected work, set a device error word and
 *   gdn_check_error reports GDN_ERR_DEVICE_DATA.  Nothing traps or hangs.
 * - Supported shapes: d_k == d_v in {64, 128}, chunk size C == 64, H >= 1.
 *   q/k/v in bf16 (d = 64 or 128) or fp32 (d = 64); beta, g and states are
 *   always fp32; output dtype bf16 (= round-to-nearest-even of the fp32
 *   result) or fp32.
 * - g must be finite (alpha = 0 is expressed as a large negative g such as
 *   -1e4, whose exp underflows to zero).
 * - Determinism: no float atomics; every (sequence, head) result depends only
 *   on that sequence's inputs, so outputs are bitwise independent of batch
 *   composition, order and padding and identical across runs.  Forward and
 *   decode (with chunk resync) produce bitwise identical outputs.
 */
#ifndef GDN_CPR_H
#define GDN_CPR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_CPR_ABI_VERSION 7

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = -1, /* null pointer, negative size, misaligned pointer, ... */
  GDN_ERR_UNSUPPORTED = -2, /* valid but not implemented: head dims, chunk size, dtype */
  GDN_ERR_WORKSPACE = -3,   /* workspace missing or smaller than the query says */
  GDN_ERR_CUDA = -4,        /* a CUDA launch or runtime call failed */
  GDN_ERR_DEVICE_DATA = -5, /* device-side validation failed (see gdn_check_error) */
  GDN_ERR_TIMEOUT = -6,     /* reserved: a bounded device-side wait gave up */
  GDN_ERR_CONTRACT = -7     /* a peer's numerical-policy digest differs from this library's */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

/* Bits of the device error word. */
#define GDN_DEVERR_CU_SEQLENS 1 /* cu_seqlens not 0-based, not nondecreasing or wrong total */
#define GDN_DEVERR_POS 2        /* a decode position outside [0, C) */
#define GDN_DEVERR_TIMEOUT 4    /* a bounded tensor-core completion wait gave up */

/* ABI version of the loaded library (GDN_CPR_ABI_VERSION it was built with). */
int gdn_cpr_abi_version(void);

/* Static string for a gdn_status value. */
const char* gdn_status_string(int status);

/*
 * Bytes of device workspace gdn_cpr_forward needs for this problem size.
 * Returns 0 for arguments gdn_cpr_forward would reject.
 */
size_t gdn_cpr_forward_workspace_bytes(int n_seqs, int64_t total_tokens, int H, int dk, int dv,
                                       int C, int in_dtype);

/*
 * gdn_cpr_forward -- CPR forward over packed variable-length sequences.
 *
 * Defines: the section "Solving the linear-attention headache" (first pass:
 * state at chunk boundaries; second pass: outputs within each chunk).
 * Chunks start at each sequence's first token and never cross a sequence
 * boundary.  Pass 1 walks the full chunks of each sequence with the chunk
 * boundary function (the same one gdn_chunk_boundary and the decode resync
 * use).  Pass 2 runs the exact per-token recurrence inside every chunk, all
 * chunks in parallel, from that chunk's boundary state.
 *
 * q, k        [total_tokens, H, dk]  in_dtype
 * v           [total_tokens, H, dv]  in_dtype
 * beta, g     [total_tokens, H]      fp32; alpha = exp(g)
 * cu_seqlens  [n_seqs + 1] int32, device; cu_seqlens[0] = 0, nondecreasing,
 *             cu_seqlens[n_seqs] = total_tokens (checked on the device)
 * h0          [n_seqs, H, dv, dk] fp32 initial states, or NULL for zeros
 * o           [total_tokens, H, dv] out_dtype (written for every token)
 * s_run_final [n_seqs, H, dv, dk] fp32 or NULL: the running state after
 *             the last token.  For a length that is a multiple of C it
 *             equals s_bnd_final; otherwise it is the recurrent state after
 *             the trailing partial chunk.  Inside a chunk the kernels keep
 *             that state as scale x mantissa (one fp32 scale per sequence
 *             and head).  With s_run_scale == NULL, s_run_final receives the
 *             state itself (scale x mantissa, rounded once).  With
 *             s_run_scale != NULL ([n_seqs, H] fp32), s_run_final receives
 *             the mantissa and s_run_scale the scale: the exact pair that
 *             gdn_cpr_decode_state_from_prefill needs for decode to continue
 *             bit for bit.
 * s_bnd_final [n_seqs, H, dv, dk] fp32 or NULL: the boundary state after the
 *             last full chunk (h0 for sequences shorter than C).
 * workspace   device scratch of at least gdn_cpr_forward_workspace_bytes;
 *             its first 4 bytes are the device error word.
 * n_seqs may be 0 and sequences may be empty.
 */
int gdn_cpr_forward(const void* q, const void* k, const void* v, int in_dtype, const float* beta,
                    const float* g, const int32_t* cu_seqlens, int n_seqs, int64_t total_tokens,
                    int H, int dk, int dv, int C, float scale, const float* h0, void* o,
                    int out_dtype, float* s_run_final, float* s_run_scale, float* s_bnd_final,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * gdn_cpr_forward_ex -- gdn_cpr_forward that also records caller-created
 * CUDA events on `stream` around its kernels, for per-kernel timing:
 * kernel_events[0] before the chunk table, [1] before the boundary prep,
 * [2] before the boundary walk, [3] before the intra-chunk fill and [4] after
 * it (an array of 5 cudaEvent_t passed as void*, or NULL for none).  The
 * computation and its bits are exactly those of gdn_cpr_forward.
 */
int gdn_cpr_forward_ex(const void* q, const void* k, const void* v, int in_dtype,
                       const float* beta, const float* g, const int32_t* cu_seqlens, int n_seqs,
                       int64_t total_tokens, int H, int dk, int dv, int C, float scale,
                       const float* h0, void* o, int out_dtype, float* s_run_final,
                       float* s_run_scale, float* s_bnd_final, void* workspace,
                       size_t workspace_bytes, void* const* kernel_events, void* stream);

/*
 * gdn_cpr_forward_noalloc -- gdn_cpr_forward for callers that cannot
 * allocate device memory.  (No counterpart on the pages: it exists for
 * callers of this library, such as a host runtime that owns the device memory
 * pool, a plugin host without a device allocator, or code that must not
 * allocate on its hot path.)
 *
 * Same arguments and results as gdn_cpr_forward, without the workspace: the
 * scratch space is a GDN_NOALLOC_SCRATCH_BYTES array compiled into the
 * library, one per GPU, kept from its first use on that device until the
 * process exits.  No cudaMalloc, cudaFree or other allocating call is made.
 * - Size limit: a problem whose gdn_cpr_forward_workspace_bytes exceeds
 *   GDN_NOALLOC_SCRATCH_BYTES is rejected with GDN_ERR_WORKSPACE before any
 *   device work.
 * - The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 * - Every call shares the array, so calls that can overlap on the GPU race;
 *   order them (one stream, or events).  Each call clears the array's error
 *   word before its kernels run.
 * - error_word: optional caller-owned device int32 (4-byte aligned); when
 *   not NULL it receives the call's device error bits (GDN_DEVERR_*),
 *   readable with gdn_check_error(error_word, ...).  An empty batch sets it to
 *   zero.  Argument errors are returned before any device work, as for
 *   gdn_cpr_forward.
 * - The array's device address is looked up in the current context on every
 *   call, so the entry point stays valid after cudaDeviceReset or a re-created
 *   primary context.
 */
#define GDN_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int gdn_cpr_forward_noalloc(const void* q, const void* k, const void* v, int in_dtype,
                            const float* beta, const float* g, const int32_t* cu_seqlens,
                            int n_seqs, int64_t total_tokens, int H, int dk, int dv, int C,
                            float scale, const float* h0, void* o, int out_dtype,
                            float* s_run_final, float* s_run_scale, float* s_bnd_final,
                            int32_t* error_word, void* stream);

/*
 * Decode state: caller-owned device arrays for n_slots sequences.
 *   s_run    [n_slots, H, dv, dk] fp32  mantissa of the running state
 *   s_scale  [n_slots, H] fp32          its scale: running state =
 *                                       s_scale x s_run (neither is read
 *                                       when pos == 0)
 *   s_bnd    [n_slots, H, dv, dk] fp32  boundary state at the start of the
 *                                       current chunk
 *   buf_k    [n_slots, H, C, dk]  in_dtype  keys of the current chunk so far
 *   buf_v    [n_slots, H, C, dv]  in_dtype  values of the current chunk so far
 *   buf_beta [n_slots, H, C] fp32, buf_g [n_slots, H, C] fp32
 *   pos      [n_slots, H] int32  tokens already in the current chunk, 0..C-1
 *                                (equal over heads; kept per head so that no
 *                                two thread blocks share a counter)
 *   error    [1] int32  device error word (GDN_DEVERR_* bits)
 *   resync   [4 + n_slots * H] int32  work list of the chunk resync inside
 *                                gdn_cpr_decode_step (scratch: all zero
 *                                before the first step; every step leaves
 *                                it zero again)
 */
typedef struct {
  float* s_run;
  float* s_scale;
  float* s_bnd;
  void* buf_k;
  void* buf_v;
  float* buf_beta;
  float* buf_g;
  int32_t* pos;
  int32_t* error;
  int32_t* resync;
  int n_slots;
} gdn_decode_state;

/*
 * gdn_cpr_decode_state_from_prefill -- hand a prefill over to decode.
 * For sequence n (slot slot_idx[n], or n when slot_idx is NULL):
 * pos = L_n mod C, the buffer receives the last pos tokens' k, v, beta, g
 * (bit copies), s_run <- s_run_final[n], s_scale <- s_run_scale[n] (1 when
 * s_run_scale is NULL), s_bnd <- s_bnd_final[n].  Decode continues bit for
 * bit from a forward only when given the forward's (s_run_final,
 * s_run_scale) pair.
 * Inputs are the packed tensors, cu_seqlens and total_tokens passed to
 * gdn_cpr_forward and the final states it produced.  A slot outside
 * [0, n_slots) or a cu_seqlens entry outside [0, total_tokens] skips that
 * sequence and sets a GDN_DEVERR_* bit in st.error.
 */
int gdn_cpr_decode_state_from_prefill(const void* k, const void* v, int in_dtype,
                                      const float* beta, const float* g,
                                      const int32_t* cu_seqlens, int n_seqs,
                                      int64_t total_tokens, int H, int dk, int dv, int C,
                                      const float* s_run_final, const float* s_run_scale,
                                      const float* s_bnd_final, const int32_t* slot_idx,
                                      gdn_decode_state st, void* stream);

/*
 * gdn_cpr_decode_step -- one batched decode step with chunk resync.
 *
 * Defines: the section "Solving the linear-attention headache" (decode runs
 * the recurrent form and re-synchronises the hidden state every chunk-size
 * tokens, so its rounding schedule matches prefill and training).
 * For each row b (slot s = slot_idx[b], or b when slot_idx is NULL) and head:
 * one recurrence step from the running state (the boundary state when
 * pos == 0) gives o[b]; the token is appended to the chunk buffer; when the
 * buffer becomes full the boundary state is advanced over the C buffered
 * tokens with the chunk boundary function and becomes the running state,
 * and pos returns to 0.
 * q, k [B, H, dk], v [B, H, dv] in_dtype; beta, g [B, H] fp32;
 * o [B, H, dv] out_dtype.  Rows must name distinct slots.
 * Two kernels run: the step (which lists the (slot, head) units whose buffer
 * became full in st.resync) and the chunk boundary of the listed units.
 * Launch shapes depend only on (B, H, dk, C) and the device, so the call can
 * be captured in a CUDA graph.
 */
int gdn_cpr_decode_step(const void* q, const void* k, const void* v, int in_dtype,
                        const float* beta, const float* g, const int32_t* slot_idx, int B, int H,
                        int dk, int dv, int C, float scale, gdn_decode_state st, void* o,
                        int out_dtype, void* stream);

/*
 * gdn_chunk_boundary -- the chunk boundary function on its own.
 * s_end[b,h] = state after applying the C tokens of chunk b, head h to
 * s_start[b,h], evaluated by the boundary schedule that gdn_cpr_forward's
 * first pass and the decode resync use (bitwise the same values).
 * s_start, s_end [B, H, dv, dk] fp32 (s_end == s_start allowed);
 * k [B, H, C, dk], v [B, H, C, dv] in_dtype; beta, g [B, H, C] fp32.
 */
int gdn_chunk_boundary(const float* s_start, const void* k, const void* v, int in_dtype,
                       const float* beta, const float* g, int B, int H, int dk, int dv, int C,
                       float* s_end, void* stream);

/*
 * gdn_recurrent_forward -- the "recurrent everywhere" forward: the per-token
 * recurrence from h0 over every token of each sequence, with no chunk
 * boundaries.
 *
 * Defines: the section "Solving the linear-attention headache" and its
 * per-layer table, whose second column runs the recurrent form for training,
 * prefill and decode alike (one rounding schedule, a serial sweep over every
 * token).  Each token runs the same step as gdn_cpr_forward's fill and
 * gdn_cpr_decode_step (the running state kept as scale x mantissa), so:
 * the first C tokens of every sequence give bitwise gdn_cpr_forward's
 * outputs, and a forward over a prefix that returns (s_final, s_final_scale)
 * continued by gdn_recurrent_decode_step gives bitwise the forward over the
 * whole sequence.
 * Arguments as gdn_cpr_forward (C is fixed at 64 and not passed; no
 * workspace): q, k [T, H, dk], v [T, H, dv] in_dtype; beta, g [T, H] fp32;
 * cu_seqlens [n_seqs + 1] int32 on the device; h0 [n_seqs, H, dv, dk] fp32
 * or NULL; o [T, H, dv] out_dtype.
 * s_final [n_seqs, H, dv, dk] fp32 or NULL: the state after each sequence's
 * last token; with s_final_scale ([n_seqs, H] fp32) it holds the mantissa and
 * s_final_scale the scale, else the state itself.
 * error_word: optional device int32 (4-byte aligned), cleared by the call;
 * cu_seqlens that do not start at 0, decrease or do not end at total_tokens
 * set GDN_DEVERR_CU_SEQLENS there and leave the offending sequences'
 * outputs unwritten.  Host-side errors are returned before any device work.
 * Supported shapes: dk = dv = 64 (bf16 or fp32 inputs) or 128 (bf16 inputs).
 */
int gdn_recurrent_forward(const void* q, const void* k, const void* v, int in_dtype,
                          const float* beta, const float* g, const int32_t* cu_seqlens,
                          int n_seqs, int64_t total_tokens, int H, int dk, int dv, float scale,
                          const float* h0, void* o, int out_dtype, float* s_final,
                          float* s_final_scale, int32_t* error_word, void* stream);

/*
 * gdn_recurrent_decode_step -- one batched step of the recurrent-everywhere
 * decode: the step of gdn_cpr_decode_step without the chunk buffer and the
 * resync.  For row b and head h: from the running state
 * s_scale[b,h] x s[b,h], one token gives o[b,h]; (s, s_scale) are updated in
 * place (mantissa and scale).
 * q, k [B, H, dk], v [B, H, dv] in_dtype; beta, g [B, H] fp32;
 * s [B, H, dv, dk] fp32; s_scale [B, H] fp32; o [B, H, dv] out_dtype.
 * A state that starts from a full state X uses (s = X, s_scale = 1).
 */
int gdn_recurrent_decode_step(const void* q, const void* k, const void* v, int in_dtype,
                              const float* beta, const float* g, int B, int H, int dk, int dv,
                              float scale, float* s, float* s_scale, void* o, int out_dtype,
                              void* stream);

/*
 * gdn_native_forward -- the chunked ("native mixed") forward: outputs from
 * each chunk's entry state by the chunkwise-parallel (UT / WY) products
 * instead of the per-token recurrence.
 *
 * Defines: the section "Solving the linear-attention headache" and its
 * per-layer table, whose first column evaluates training and prefill
 * chunkwise in parallel while decode runs the recurrent form (the layout
 * whose prefill and decode round differently).  With G the chunk's
 * cumulative log-decay and U = T diag(beta) V - T diag(beta e^G) K S^T
 * (T = (I + A)^{-1} as in gdn_chunk_boundary):
 *     o_i = scale (e^{G_i} S q_i + sum_{j <= i} e^{G_i - G_j} (q_i . k_j) u_j)
 * The entry states S are gdn_cpr_forward's first-pass boundary states
 * (the same kernels); the output products run on the tensor cores with
 * two-term bf16 splits of the non-bf16 operands, so o agrees with
 * gdn_cpr_forward within the forward's bounds but not bit for bit.
 * Arguments as gdn_cpr_forward (same workspace size); s_final receives the
 * state after the last token (the state itself) and s_bnd_final the last
 * boundary state.  Supported shape: dk = dv = 128 with bf16 inputs
 * (GDN_ERR_UNSUPPORTED otherwise).  kernel_events: NULL, or 5 cudaEvent_t
 * recorded before the chunk table, the boundary prep, the walk, the output
 * products and after them.
 */
int gdn_native_forward(const void* q, const void* k, const void* v, int in_dtype,
                       const float* beta, const float* g, const int32_t* cu_seqlens, int n_seqs,
                       int64_t total_tokens, int H, int dk, int dv, int C, float scale,
                       const float* h0, void* o, int out_dtype, float* s_final,
                       float* s_bnd_final, void* workspace, size_t workspace_bytes,
                       void* const* kernel_events, void* stream);

/*
 * Bytes of device workspace gdn_cpr_backward needs for this problem size.
 * Returns 0 for arguments gdn_cpr_backward would reject.
 */
size_t gdn_cpr_backward_workspace_bytes(int n_seqs, int64_t total_tokens, int H, int dk, int dv,
                                        int C, int in_dtype);

/*
 * gdn_cpr_backward -- reverse mode of gdn_cpr_forward: the gradients of a
 * loss L(o, S_final) with respect to q, k, v, beta, g and h0, given dL/do and
 * dL/dS_final.  S_final is the state after each sequence's last token.
 *
 * Defines: the trainer's forward plus backward of the section "Solving the
 * linear-attention headache" (its timing table has a row for it); the pages
 * give no formulas, so the gradients are those of the recurrence
 * S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 * o_t = scale S_t q_t, alpha_t = exp(g_t).
 * Schedule: the forward's first pass runs again (boundary states); an
 * adjoint recurrence runs over each sequence, last token first (row-parallel,
 * like the state); each chunk's update vectors u are recomputed from its
 * boundary state (bf16 inputs: in product form, U = T diag(beta)(V -
 * diag(e^G) K S_a^T); fp32 inputs: with the forward's per-token step); each
 * chunk's dq and dk, and with bf16 inputs its dbeta and dg, come from
 * products of C x C and C x d matrices.  Every reduction has a fixed order,
 * so repeated calls return identical bits.
 *
 * Inputs:  q, k, v, beta, g, cu_seqlens, n_seqs, total_tokens, H, dk, dv, C,
 *          scale, h0 exactly as for gdn_cpr_forward.
 *   d_o       [total_tokens, H, dv] in_dtype: dL/do
 *   ds_final  [n_seqs, H, dv, dk] fp32 dL/dS_final, or NULL for zeros
 * Outputs (fp32, written for every token; caller-owned device memory):
 *   d_q, d_k  [total_tokens, H, dk]
 *   d_v       [total_tokens, H, dv]
 *   d_beta, d_g [total_tokens, H]
 *   d_h0      [n_seqs, H, dv, dk] dL/dh0 (whether or not h0 is NULL), or
 *             NULL to skip it
 * workspace: device scratch of at least gdn_cpr_backward_workspace_bytes
 *   bytes, 16-byte aligned.  Its first 4 bytes are the device error word.
 *   Its first gdn_cpr_forward_workspace_bytes bytes are laid out as the
 *   forward's workspace, so the same buffer can serve a gdn_cpr_forward call.
 * flags: 0, or GDN_BWD_REUSE_FORWARD: the workspace was last written by a
 *   gdn_cpr_forward call with the same q, k, v, beta, g, cu_seqlens, h0,
 *   shapes and C (a trainer's forward followed by its backward); the first
 *   pass is then not run again, and the gradients are bit for bit those of a
 *   call without the flag.  The library cannot check that promise; gradients
 *   of a different batch's boundary states are wrong, not an error.
 * Pointers to device arrays of 16-byte rows must be 16-byte aligned.
 * Status: as gdn_cpr_forward (GDN_ERR_INVALID_ARG also for unknown flags);
 * invalid cu_seqlens set GDN_DEVERR_CU_SEQLENS in the error word and leave
 * the outputs unwritten.
 */
#define GDN_BWD_REUSE_FORWARD 1
int gdn_cpr_backward(const void* q, const void* k, const void* v, int in_dtype,
                     const float* beta, const float* g, const int32_t* cu_seqlens, int n_seqs,
                     int64_t total_tokens, int H, int dk, int dv, int C, float scale,
                     const float* h0, const void* d_o, const float* ds_final, float* d_q,
                     float* d_k, float* d_v, float* d_beta, float* d_g, float* d_h0,
                     void* workspace, size_t workspace_bytes, int flags, void* stream);

/*
 * gdn_cpr_backward_ex -- gdn_cpr_backward that also records caller-created
 * CUDA events on `stream` around its kernels, for per-kernel timing:
 * kernel_events[0] before the first pass (recorded even when it is reused),
 * [1] before the adjoint scan, [2] before the per-chunk state recomputation,
 * [3] before the chunk products and [4] after them (an array of 5
 * cudaEvent_t passed as void*, or NULL for none).  The computation and its
 * bits are exactly those of gdn_cpr_backward.
 */
int gdn_cpr_backward_ex(const void* q, const void* k, const void* v, int in_dtype,
                        const float* beta, const float* g, const int32_t* cu_seqlens,
                        int n_seqs, int64_t total_tokens, int H, int dk, int dv, int C,
                        float scale, const float* h0, const void* d_o, const float* ds_final,
                        float* d_q, float* d_k, float* d_v, float* d_beta, float* d_g,
                        float* d_h0, void* workspace, size_t workspace_bytes, int flags,
                        void* const* kernel_events, void* stream);

/*
 * gdn_check_error -- synchronise `stream`, read the device error word at
 * `error_word` (the forward workspace, or a decode state's `error`), clear
 * it, and return GDN_OK or GDN_ERR_DEVICE_DATA.  If bits_out is not NULL it
 * receives the GDN_DEVERR_* bits that were set.
 */
int gdn_check_error(void* error_word, int32_t* bits_out, void* stream);

/*
 * Contract digests of the CPR region (host only, no device work).
 *
 * Defines: "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI
 * Training Runs", section "The execution contract": a contract pins every
 * choice that can move bits and carries three SHA-256 identity digests
 * (semantic equivalence, numerical policy, deployment settings that do not
 * affect bits); engines whose numerical policies differ refuse to run
 * together.  Each digest is the SHA-256 (FIPS 180-4) of a canonical text
 * descriptor of this library's region for one (in_dtype, out_dtype, dk, dv,
 * C): what it computes (semantic); every choice that fixes its bits, i.e.
 * dtypes, shapes, the step and boundary schedules and their versions, the
 * operand splits, the MMA shapes and the compile flags (numerical policy);
 * and settings that do not change bits such as the ABI version and the SM
 * count of the current device (deployment).
 * Status: GDN_ERR_INVALID_ARG for an unknown kind or a NULL output,
 * GDN_ERR_UNSUPPORTED for a shape or dtype the library does not run.
 */
typedef enum {
  GDN_DIGEST_SEMANTIC = 0,
  GDN_DIGEST_POLICY = 1,
  GDN_DIGEST_DEPLOYMENT = 2
} gdn_digest_kind;

/* The descriptor text (NUL-terminated) into buf[buf_bytes]; *len_out = its
 * length without the NUL.  buf == NULL only queries the length;
 * GDN_ERR_INVALID_ARG when buf is too small. */
int gdn_cpr_contract_descriptor(int kind, int in_dtype, int out_dtype, int dk, int dv, int C,
                                char* buf, size_t buf_bytes, size_t* len_out);

/* out32[32] = SHA-256 of that descriptor. */
int gdn_cpr_contract_digest(int kind, int in_dtype, int out_dtype, int dk, int dv, int C,
                            uint8_t* out32);

/* Refuse to mix: GDN_OK when peer_policy32[32] equals this library's
 * numerical-policy digest for the shape, GDN_ERR_CONTRACT when it differs. */
int gdn_cpr_contract_check(const uint8_t* peer_policy32, int in_dtype, int out_dtype, int dk,
                           int dv, int C);

/* out32[32] = SHA-256 of data[n] (the hash the digests use). */
int gdn_sha256(const void* data, size_t n, uint8_t* out32);

/*
 * gdn_selftest_bounded_wait -- exercise the give-up path of the boundary
 * walk's bounded waits (this library's own safeguard; the pages have no
 * counterpart).  One block allocates tensor memory as the walk does, waits
 * `polls` polls (1 .. 2^22) on a completion barrier that nothing arrives at,
 * sets GDN_DEVERR_TIMEOUT in *error_word (device int32), frees the tensor
 * memory and returns; the context stays usable.  Asynchronous on `stream`;
 * read the bit with gdn_check_error.
 */
int gdn_selftest_bounded_wait(int polls, int32_t* error_word, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_CPR_H */
