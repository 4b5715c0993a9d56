/*
 * gdn_pik.h -- parallelism-invariant K-leaf GEMM (sm_100a, tcgen05).
 *
 * Defines: "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI
 * Training Runs", section "Making kernels parallelism-invariant" and its
 * reduction-tree figure.  The K dimension of a GEMM is cut into contiguous
 * leaves, each leaf is a tensor-core product accumulated in fp32, the leaves
 * are combined by one fixed binary tree, and each rank always owns the same
 * contiguous leaves, so the result does not depend on the number of ranks.
 * This library runs the single-GPU form: the ranks are emulated on one GPU
 * and their partials never leave it.
 *
 * Status codes are those of gdn_cpr.h (GDN_OK, GDN_ERR_*).
 */
#ifndef GDN_PIK_H
#define GDN_PIK_H

#include <stddef.h>
#include <stdint.h>

#include "gdn_cpr.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Bytes of device workspace gdn_pik_gemm needs (0 when it needs none, and
 * for arguments it would reject).
 */
size_t gdn_pik_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_leaves, int n_ranks);

/*
 * gdn_pik_gemm -- C = A B^T, with K cut into n_leaves contiguous leaves of
 * K / n_leaves (leaf l covers k in [l K/L, (l+1) K/L)).  Each leaf is a
 * sum of tcgen05 MMAs (M 128, K 16 each) in ascending k with fp32
 * accumulation in tensor memory; the leaves are combined by the balanced
 * binary tree (level by level, neighbours 2i and 2i+1, left operand first,
 * fp32 round to nearest).
 *
 * n_ranks emulates that many ranks, rank r owning leaves
 * [r L/R, (r+1) L/R): the work is cut into that rank layout and the group
 * sums are combined above it.  The bits of C are the same for every n_ranks
 * (and for every grouping of the leaves the library chooses).
 *
 * A          [M, K] bf16, row-major (K innermost), device, 16-byte aligned
 * B          [N, K] bf16, row-major (K innermost), device, 16-byte aligned
 * C          [M, N] fp32, row-major, device, 16-byte aligned (written)
 * n_leaves   L: a power of two, 1 .. 64; K must be a multiple of 64 L
 * n_ranks    R: a power of two dividing L
 * N          a multiple of 16; M any size (M = 0 or N = 0: nothing to do;
 *            K = 0: C is set to zero and A, B are not read)
 * workspace  gdn_pik_workspace_bytes bytes of device memory (may be NULL
 *            when that is 0), 16-byte aligned
 * error_word device int32, 4-byte aligned: GDN_DEVERR_TIMEOUT is OR-ed in
 *            when a bounded wait for the tensor core gives up (C is then
 *            not written for that tile); read it with gdn_check_error.
 * stream     cudaStream_t, or NULL for the default stream.
 * Status: GDN_ERR_INVALID_ARG for negative sizes, NULL or misaligned
 * pointers; GDN_ERR_UNSUPPORTED for L, R, N or K outside the rules above;
 * GDN_ERR_WORKSPACE for a missing or short workspace; GDN_ERR_CUDA for a
 * launch error.
 */
int gdn_pik_gemm(const void* A, const void* B, float* C, int64_t M, int64_t N, int64_t K,
                 int n_leaves, int n_ranks, void* workspace, size_t workspace_bytes,
                 int32_t* error_word, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_PIK_H */
