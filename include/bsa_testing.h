/*
 * bsa_testing.h — test-only entry point of libbsa.so. Not part of the BSA
 * method and not for production use.
 */
#ifndef BSA_TESTING_H
#define BSA_TESTING_H

#include "bsa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bsa_fine_attention on the tensor-core kernel (bf16, block 64, head_dim 64
 * only) with the value-tile copy of pipeline step `withhold_v_step` of the
 * first pipeline deliberately not issued. The wait for that copy expires
 * after its bound (about 2 s); the kernel then records BSA_ERR_TIMEOUT in
 * *status_word (required, device, zero before the call), stops, drains its
 * own copies and MMAs, frees its tensor memory and returns. `out` is left
 * incomplete. Lets a test check the timeout path without faulting the GPU.
 * Returns BSA_ERR_UNSUPPORTED for shapes the tensor-core kernel does not take.
 */
BSA_API bsa_status bsa_testing_fine_attention_withhold(const bsa_config *cfg, const void *q, const void *k,
                                                       const void *v, const float *gates,
                                                       const float *o_cg_block, const int32_t *sel_idx,
                                                       void *out, uint32_t *status_word,
                                                       int64_t withhold_v_step, cudaStream_t stream);

/*
 * y[i] = 2^x[i] (n device floats) as the fine-attention kernel's softmax forms
 * it: poly != 0 takes the FMA-pipe route (range reduction and a degree-3
 * minimax polynomial), poly == 0 the exp unit (ex2.approx). Lets a test hold
 * the polynomial to its error bound against exact 2^x and the exp unit.
 */
BSA_API bsa_status bsa_testing_exp2(const float *x, float *y, int64_t n, int32_t poly, cudaStream_t stream);

/*
 * Tensor-pipe rate microbenchmark: one CTA, `warps` (1, 2 or 4) warps each with
 * one thread issuing 256 back-to-back tcgen05.mma (kind::f16, bf16 zero
 * operands in shared memory, K = 16) of an m x n tile (m 64 or 128, n 64, 128
 * or 256) into its own tensor-memory columns, then waiting (bounded) for them.
 * cycles (device, 8-byte aligned, `warps` entries) receives each warp's clock
 * cycles from its first issue to completion, or -1 if the wait expired. The
 * multiply-add rate of the SM is m*n*16*256*warps / max(cycles). Used to
 * measure the M = 64 ceiling of the fine-attention kernel (an M = 64 tile
 * drives half of the tensor datapath). Returns BSA_ERR_INVALID_ARG for other
 * shapes or warp counts.
 */
BSA_API bsa_status bsa_testing_mma_rate(int32_t m, int32_t n, int32_t warps, int64_t *cycles, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_TESTING_H */
