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

#ifdef __cplusplus
}
#endif

#endif /* BSA_TESTING_H */
