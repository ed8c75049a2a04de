/*
 * liblstm_testing.h -- test hooks of liblstm.  Not part of the LSTM API: they
 * expose the library's internal kernels so that tests can check each one in
 * isolation against a library routine.
 */
#ifndef LIBLSTM_TESTING_H
#define LIBLSTM_TESTING_H

#include <stddef.h>

/*
 * Environment variables.  The library reads exactly these, at every call
 * (nothing is cached); each is unset by default, and any other value than
 * the one shown means "unset".  They exist for tests, comparison runs and
 * profiling, never for results: every setting gives results within the same
 * tolerance.
 *
 *   LSTM_FORCE_SIMT=1      run every step on the CUDA-core kernels (no tensor
 *                          cores, no persistent kernels).
 *   LSTM_FWD_FUSED_X=0     do not run the forward kernel with the input
 *                          projection fused into the recurrence; the forward
 *                          then needs the Gx workspace
 *                          (lstm_fwd_workspace_size_max).
 *   LSTM_BWD_TMEM_W=0      do not run the backward kernel with W_h^T in tensor
 *                          memory (the older cluster kernels run instead).
 *   LSTM_BWD_STREAMS=1     run that backward kernel with one batch stream per
 *                          group instead of two decoupled streams.
 *   LSTM_PERSIST=0         run the CUDA-core recurrences (fp32, and 16-bit
 *                          shapes off the tensor-core grids) as one launch
 *                          per step instead of one persistent launch.
 *   LSTM_PERSIST_KS=n      split those persistent recurrences' K axis over
 *                          clusters of n CTAs only (1, 2, 4 or 8; 1 = no
 *                          split).  Default: the split with the lowest
 *                          estimated step time that fits and is co-resident;
 *                          when n does not fit, the per-step kernels run.
 *   LSTM_STACK_WAVE=0      run the layers of lstm_stack_fwd / lstm_stack_bwd
 *                          one after another instead of as a layer wavefront
 *                          (two layers' time chunks side by side on half the
 *                          SMs each).
 *   LSTM_STACK_CHUNKS=n    chunks per layer of that wavefront (1..8; 1 = each
 *                          layer in one launch, after the layer below it).
 *                          Default: min(8, T / 8), and no wavefront below 2.
 *   LSTM_BWD_CHUNKS=n      run the tensor-core backward recurrence in n
 *                          reverse-time chunks (1..16; 1 = one launch, dW / dx
 *                          after it).  Default: min(6, T / 16), 1 below T = 32.
 *   LSTM_LAUNCH_NONCOOP=1  launch the persistent cluster kernels without the
 *                          cooperative attribute, after the same co-residency
 *                          check (profilers cannot replay cooperative cluster
 *                          launches).  Taken automatically when a profiler
 *                          or sanitizer is attached: Nsight Compute sets
 *                          NV_COMPUTE_PROFILER_PERFWORKS_DIR in the profiled
 *                          process, injection-based tools set
 *                          CUDA_INJECTION64_PATH.
 */

#ifdef __cplusplus
extern "C" {
#endif

/*
 * C[M][N] (float, row stride ldc) = A B^T (+ bias[n]) through the tcgen05 / TMA
 * GEMM core that the input projection, dW and dx use, with bf16 operands.
 *   a_mn_major = 0: A is [M][K] row-major with row stride lda (K-major)
 *   a_mn_major = 1: A is [K][M] row-major with row stride lda (MN-major)
 *   b_mn_major = 0: B is [N][K] row-major with row stride ldb (K-major)
 *   b_mn_major = 1: B is [K][N] row-major with row stride ldb (MN-major)
 * bias is bf16 [N] or NULL.  Device pointers, 16-byte aligned; lda and ldb
 * multiples of 8.  ws holds at least 256 bytes (the status word).
 * Returns an LSTM_* status code (see liblstm.h).
 */
int lstm_test_tc_gemm(int M, int N, int K, const void *A, long long lda, int a_mn_major,
                      const void *B, long long ldb, int b_mn_major, const void *bias, float *C,
                      long long ldc, void *ws, size_t ws_bytes, void *stream);

/*
 * Failure-detection hook for the persistent recurrent kernels: from now on,
 * CTA `skip_cta` of every persistent launch never signals its step barrier
 * (-1 turns that off), and every device-side wait gives up after `wait_ns`
 * nanoseconds (<= 0 restores the default of 2 s).  A wait that gives up records
 * LSTM_ERR_TIMEOUT in the workspace status word and the kernel returns; nothing
 * faults.  Process-wide, not thread-safe.
 */
int lstm_test_set_wait_fault(int skip_cta, long long wait_ns);

/*
 * Which recurrent kernel the most recent lstm_fwd / lstm_bwd of this process
 * used: 0 = one CUDA-core launch per step (fp32, or shapes off the tensor-core
 * grid), 5 = the persistent CUDA-core kernel for those (all steps in one
 * launch), 1 = persistent tensor-core kernel with K resident per CTA, 2 = persistent cluster
 * kernel with K split across the CTAs of a cluster, 3 = the cluster kernel
 * with the weights held in tensor memory (forward: with the input projection
 * contracted inside the recurrence), 4 = (backward) that kernel with two
 * batch streams per group, each with its own TMA producer, MMA issuer and
 * epilogue warpgroup; -1 = none yet.
 */
int lstm_test_last_paths(int *fwd_path, int *bwd_path);

/*
 * Chunks per layer of the layer wavefronts that the most recent
 * lstm_stack_fwd and lstm_stack_bwd of this process ran (0: its layers ran
 * one after another; -1: none yet).
 */
int lstm_test_last_stack_chunks(int *fwd_chunks, int *bwd_chunks);

/*
 * Cluster size (the number of CTAs that split the contraction's K axis) of
 * the persistent CUDA-core forward and backward recurrences that this process
 * launched last (0: none yet).
 */
int lstm_test_last_persist_split(int *fwd_ks, int *bwd_ks);

/*
 * Reverse-time chunking of the tensor-core backward: the number of chunk
 * launches a call over `T` steps uses (after LSTM_BWD_CHUNKS), and the first
 * epilogue iteration of chunk `c` (c = nch gives T).  Host logic only; no GPU
 * needed.
 */
int lstm_test_bwd_chunks(int T);
int lstm_test_chunk_bound(int T, int nch, int c);

#ifdef __cplusplus
}
#endif

#endif /* LIBLSTM_TESTING_H */
