/*
 * attn_ablation.h — entry points that exist only in the ablation builds of libattn.so
 * (libattn_abl.so, libattn_abl_sw4.so; built by tiled_attention_14_b200/build.py with
 * ATTN_ABLATION).  They measure two choices of the online softmax that the page
 * "FlashAttention 4: Γρηγορότερη και Αποδοτική σε Μνήμη Προσοχή για LLMs" describes:
 * the rescale threshold (section "Έξυπνος επανακανονισμός Softmax στο Διαδίκτυο": the
 * running maximum is only raised when a new maximum exceeds it by a margin, which the page
 * says cuts rescaling about tenfold) and the software exp2 on the FMA units (section
 * "Αποκορύφωση Λογισμικού μέσω Πυρήνων CUDA").  Every other entry point of attn.h is
 * present and behaves as in the product build, except that the attention kernels read the
 * threshold from device memory and count rescales.  Not for production use.
 */
#ifndef ATTN_ABLATION_H_
#define ATTN_ABLATION_H_

#include "attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Sets the rescale threshold tau (log2 units, 0 <= tau <= 8 so that P <= 256 fits bf16 and
 * e4m3; tau = 0 is the classic online softmax that rescales on every new maximum) for the
 * current device and zeroes the counters.  ATTN_ERR_INVALID for tau outside [0, 8]. */
ATTN_API int attn_ablation_set(float tau);

/* Synchronises the device and reads the counters since attn_ablation_set:
 * out[0] = (row, key tile) softmax steps that rescaled O and the row sum,
 * out[1] = (row, key tile) steps of rows that had seen at least one visible key. */
ATTN_API int attn_ablation_counts(unsigned long long* out);

/* 0 if every exponential runs on the MUFU unit; n if one element pair in n uses the
 * software exp2 (a Cody-Waite split and a cubic on the FMA pipes). */
ATTN_API int attn_ablation_sw_exp_every(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_ABLATION_H_ */
