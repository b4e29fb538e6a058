/*
 * attn.h — C-ABI of libattn.so: fused scaled-dot-product attention forward for
 * NVIDIA B200 (sm_100a), with the FlexAttention variants and an FP8 e4m3 path.
 *
 * What the calls compute
 * ----------------------
 *   O = softmax(score_mod(scale * Q K^T) masked by mask_mod) V,  LSE = ln sum exp(...)
 * tile by tile with an online (running max / running sum) softmax, so the S x S score
 * matrix never reaches HBM.  Definition: page "FlashAttention 4: Γρηγορότερη και
 * Αποδοτική σε Μνήμη Προσοχή για LLMs", sections "Εισαγωγή" (softmax of Q K^T times V)
 * and "Γιατί οι πυρήνες προσοχής ..." (tiles staged on chip, only the running max and
 * sum kept per query row).  Variants: page "PyTorch's FlexAttention mit
 * FlashAttention-4 ist ein Game-Changer", intro (ALiBi, sliding window, document
 * masking, soft-capping) and section "Leistung und Validierung" (causal).  Block
 * sparsity: same page, section "Aktuelle Einschränkungen".  FP8 with block
 * quantisation: page "FlashAttention-3: Rekordverdächtige Geschwindigkeit ...",
 * section "Analyse".
 *
 * Conventions shared by every call
 * --------------------------------
 * - Tensors are caller-owned DEVICE memory, contiguous, layout [B, H, S, D] (row i of
 *   (b, h) at element offset ((b*H + h)*S + i)*D).  The library never frees or keeps
 *   them and writes only the output arguments.
 * - Pointers must be 16-byte aligned.  D is 64 or 128.  B, H, Sq, Sk >= 1 and
 *   Sq, Sk <= ATTN_MAX_SEQ.
 * - Causal alignment is bottom-right: query row i sits at key position
 *   i' = i + (Sk - Sq).  CAUSAL keeps j <= i'.  WINDOW (width W >= 1) keeps
 *   i' - j < W together with CAUSAL, |i' - j| < W without it.  DOC keeps
 *   doc_ids[b, i] == doc_ids[b, j] and needs Sq == Sk.  The bits may be combined.
 * - score_mod order: t = scale * q.k; if softcap > 0: t = softcap * tanh(t / softcap);
 *   if alibi_slopes: t += alibi_slopes[h] * (j - i').
 * - A query row that sees no key gets O = 0 and LSE = -inf.  LSE is natural-log.
 * - Argument errors are returned synchronously and nothing is launched.  Launch
 *   failures return ATTN_ERR_CUDA.  Errors raised inside a kernel (a bounded wait
 *   that ran out) are recorded in a per-device status word read by attn_get_status.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *   stream).  The device must be compute capability 10.0 (B200); anything else gets
 *   ATTN_ERR_UNSUPPORTED.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = -1,      /* bad argument; nothing launched */
  ATTN_ERR_UNSUPPORTED = -2,  /* device is not sm_100 */
  ATTN_ERR_CUDA = -3,         /* a CUDA runtime/driver call or launch failed */
  ATTN_ERR_TIMEOUT = -4,      /* a kernel's bounded wait ran out (from attn_get_status) */
  ATTN_ERR_NOMEM = -5,        /* workspace allocation failed */
  ATTN_ERR_CHECK = -6         /* debug build only: a TMA or TMEM bounds check failed in a kernel */
} attn_status;

enum {
  ATTN_MASK_NONE = 0,
  ATTN_MASK_CAUSAL = 1,
  ATTN_MASK_WINDOW = 2,
  ATTN_MASK_DOC = 4
};

/* Tile-map geometry and entry format (see attn_tile_map_build). */
enum {
  ATTN_MAP_BLOCK_Q = 256,     /* query rows per map block: two 128-row query tiles */
  ATTN_MAP_TILE_K = 128,      /* key columns per key tile */
  ATTN_TILE_EMPTY = 0,
  ATTN_TILE_PARTIAL = 1,
  ATTN_TILE_FULL = 2
};
#define ATTN_MAP_ENTRY(kt, c0, c1) ((uint32_t)(kt) | ((uint32_t)(c0) << 24) | ((uint32_t)(c1) << 26))

#define ATTN_MAX_SEQ (1 << 20)

/*
 * attn_fwd — BF16 attention forward.
 *   q        bf16 [B,H,Sq,D]   (device, read)
 *   k, v     bf16 [B,H,Sk,D]   (device, read)
 *   o        bf16 [B,H,Sq,D]   (device, written)
 *   lse      fp32 [B,H,Sq]     (device, written; natural log)
 *   scale    finite, > 0 (usually 1/sqrt(D))
 *   mask_kind  OR of ATTN_MASK_* bits
 *   window   W >= 1, used iff the WINDOW bit is set
 *   softcap  <= 0 turns soft-capping off; otherwise finite
 *   alibi_slopes  device fp32 [H], or NULL for no ALiBi
 *   doc_ids  device int32 [B,Sk], required iff the DOC bit is set (then Sq == Sk)
 * With the DOC bit the call builds a tile map in a stream-ordered workspace
 * (cudaMallocAsync / cudaFreeAsync on `stream`; B <= 65535) and then runs the attention kernel;
 * fully masked tiles are skipped.  CAUSAL and WINDOW tile ranges are computed in the
 * kernel and need no workspace.  Accumulation is fp32; P is rounded to bf16 for P.V.
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int H, int Sq, int Sk, int D, float scale,
             int mask_kind, int window, float softcap,
             const float* alibi_slopes, const int* doc_ids, void* stream);

/*
 * attn_fwd_gqa — attn_fwd with grouped-query / multi-query heads: H query heads share
 * H_kv key/value heads (H_kv divides H; query head h reads key/value head h / (H / H_kv);
 * H_kv = 1 is multi-query attention, H_kv = H is attn_fwd).  Grouped heads: page
 * "FlashAttention 4: ...", section "Συμβατότητα και τρέχουσα κατάσταση".
 *   q  bf16 [B,H,Sq,D];  k, v  bf16 [B,H_kv,Sk,D];  o, lse and every other argument as
 *   attn_fwd (alibi_slopes has H entries, one per query head).
 */
ATTN_API int attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int H_kv, int Sq, int Sk, int D, float scale,
                          int mask_kind, int window, float softcap,
                          const float* alibi_slopes, const int* doc_ids, void* stream);

/*
 * attn_fwd_pair — attn_fwd_gqa computed by the kernel that runs each 256-row query block on a
 * cluster of two CTAs on two SMs: the pair MMA (tcgen05 cta_group::2, M = 256) with each CTA
 * holding 128 query rows, half of every K/V tile and two S buffers in its tensor memory, so
 * that S of the next key tile overlaps the softmax of this one.  The page "Hardware-Aware FP4
 * FlashAttention-4" (paragraph on on-chip storage) names the full on-chip storage that keeps
 * stages from overlapping; the FlexAttention page names the 256x128 Blackwell tile (section
 * "Aktuelle Einschränkungen").  BF16 with D = 128 only (other D: ATTN_ERR_INVALID); same
 * arguments, layouts, masks and results (within the same tolerance) as attn_fwd_gqa.
 * Measured on B200 it is slower than attn_fwd (about 0.8x), which is why attn_fwd does not
 * use it; it is kept as a tested alternative.  Launched as 2-CTA clusters; every wait is
 * bounded as in attn_fwd.
 */
ATTN_API int attn_fwd_pair(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int H_kv, int Sq, int Sk, int D, float scale,
                           int mask_kind, int window, float softcap,
                           const float* alibi_slopes, const int* doc_ids, void* stream);

/*
 * attn_fwd_varlen — attention over packed variable-length sequences, without padding
 * (page "FlashAttention 4: ...", section "Συμβατότητα και τρέχουσα κατάσταση").
 * Sequence s owns query tokens cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 and key tokens
 * cu_seqlens_k[s] .. cu_seqlens_k[s+1]-1 and attends only within itself; masks, causal
 * alignment (bottom-right) and ALiBi positions are per sequence, as if each sequence were
 * its own batch entry.  Token-major tensors:
 *   q  bf16 [total_q, H, D];  k, v  bf16 [total_k, H_kv, D]  (device, read)
 *   o  bf16 [total_q, H, D];  lse  fp32 [H, total_q]         (device, written)
 *   cu_seqlens_q / cu_seqlens_k  device int32 [nseq + 1], non-decreasing, starting at 0
 *   max_seqlen_q / max_seqlen_k  upper bounds of the sequence lengths (the work is laid
 *   out for them); total_q / total_k >= 1 the token counts of the tensors.
 * mask_kind: CAUSAL and WINDOW (DOC is rejected: the sequences are the documents).  Other
 * arguments as attn_fwd_gqa.  The offsets live in device memory, so the host cannot check
 * them: a sequence that leaves its tensor or exceeds a stated maximum is skipped (its
 * outputs are not written) and ATTN_ERR_INVALID is recorded for attn_get_status.  Key rows
 * past a sequence's end are masked; their V values are multiplied by 0, so they must be
 * finite (the tokens of the neighbouring sequence, or TMA zero fill past total_k).
 */
ATTN_API int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                             const int* cu_seqlens_q, const int* cu_seqlens_k, int nseq,
                             int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                             int H, int H_kv, int D, float scale,
                             int mask_kind, int window, float softcap,
                             const float* alibi_slopes, void* stream);

/*
 * attn_fwd_noalloc — attn_fwd that allocates no device memory.  (An addition of this
 * library; the method itself has no counterpart for it.)
 * Meant for callers that cannot allocate during a call: code inside a framework whose own
 * caching allocator owns device memory, serving loops where an allocation or free could
 * synchronise the device mid-request, and programs with a fixed memory budget.  The tile
 * map of the DOC bit goes into a library-owned static device array of
 * ATTN_NOALLOC_SCRATCH_BYTES (4 MiB) per device, held until the process exits; a map that
 * needs more (bytes ~ 4*B*ceil(Sq/256)*ceil(Sk/128)) returns ATTN_ERR_INVALID, nothing
 * launched.  Without the DOC bit no scratch is used at all.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress, with that device current),
 * so make that first call before any stream capture.  With CUDA's default lazy module
 * loading that first call also loads the library's device code onto the device, and
 * loading allocates device memory for it (the 4 MiB array included): the guarantee of
 * no allocation holds from the second call on, so make one warm-up call per device
 * first (or set CUDA_MODULE_LOADING=EAGER, which loads everything at context creation).
 * A DOC call with B > 65535 returns ATTN_ERR_INVALID.  All calls on one device share the
 * array: calls whose kernels may overlap on the GPU race on it and must be ordered (one
 * stream, or events).  Arguments, outputs and errors as attn_fwd (BF16, D = 64 or 128).
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (4 << 20)
ATTN_API int attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int H, int Sq, int Sk, int D, float scale,
                              int mask_kind, int window, float softcap,
                              const float* alibi_slopes, const int* doc_ids, void* stream);

/*
 * attn_bwd — attention backward: dQ, dK, dV of the forward above (same arguments, score_mod
 * and masks; grouped-query heads as attn_fwd_gqa) from the forward's inputs, its output O
 * and log-sum-exp LSE, and the output gradient dO.  The pages compare FA4's backward with
 * cuDNN's and note that block-sparse backward runs are not deterministic (page "PyTorch's
 * FlexAttention mit FlashAttention-4 ist ein Game-Changer", sections "Leistung und
 * Validierung" and "Aktuelle Einschränkungen"); this one is: no floating-point atomics, a
 * fixed accumulation order, bitwise identical results run to run.  ALiBi slopes get no
 * gradient (captured tensors get none, same section).
 *   q, o, dout  bf16 [B,H,Sq,D];  k, v  bf16 [B,H_kv,Sk,D];  lse  fp32 [B,H,Sq] (natural log,
 *   -inf for rows that saw no key)                                (device, read)
 *   dq  bf16 [B,H,Sq,D];  dk, dv  bf16 [B,H_kv,Sk,D]              (device, written)
 * dK and dV of a key/value head sum over the query heads that share it.  Internally fp32:
 * P and dS are rounded to bf16 as tensor-core operands.  Three launches on `stream` (row
 * sums of dO*O and log2-scaled LSE into a stream-ordered workspace, then the dK/dV kernel,
 * then the dQ kernel).  Other arguments and errors as attn_fwd_gqa.
 */
ATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv,
                      int B, int H, int H_kv, int Sq, int Sk, int D, float scale,
                      int mask_kind, int window, float softcap,
                      const float* alibi_slopes, const int* doc_ids, void* stream);

/*
 * attn_tile_map_build — classify every (256-row query block, 128-column key tile) pair
 * as EMPTY, PARTIAL or FULL under the mask and list the non-empty key tiles.
 *   counts   device int32 [B, ceil(Sq/256)]               (written)
 *   entries  device uint32 [B, ceil(Sq/256), ceil(Sk/128)] (written; only the first
 *            counts[b,qb] entries of each row are meaningful)
 * Entry = ATTN_MAP_ENTRY(kt, class of query tile 0, class of query tile 1), listed in
 * increasing kt; a key tile is listed iff one of the two classes is not EMPTY.  EMPTY
 * means no visible pair among valid rows (i < Sq) and keys (j < Sk); FULL means all
 * 128 keys of the tile are valid and visible to every valid row; PARTIAL otherwise.
 * The classification is exact (every pair is tested).  Mask arguments as attn_fwd;
 * doc_ids may be NULL unless the DOC bit is set.
 */
ATTN_API int attn_tile_map_build(int* counts, uint32_t* entries, int B, int Sq, int Sk,
                        int mask_kind, int window, const int* doc_ids, void* stream);

/*
 * attn_fwd_with_map — attn_fwd driven by a caller-supplied tile map (same format as
 * attn_tile_map_build writes; same for every head).  The kernel visits exactly the
 * listed key tiles, applies the element mask on PARTIAL tiles and trusts FULL tiles
 * to need none.  A map that lists every key tile as PARTIAL computes the same result
 * as skipping (fully masked tiles add exact zeros).  Other arguments as attn_fwd.
 */
ATTN_API int attn_fwd_with_map(const void* q, const void* k, const void* v, void* o, float* lse,
                      int B, int H, int Sq, int Sk, int D, float scale,
                      int mask_kind, int window, float softcap,
                      const float* alibi_slopes, const int* doc_ids,
                      const int* counts, const uint32_t* entries, void* stream);

/*
 * attn_quantize_e4m3 — per-block FP8 quantiser (FP8 with block quantisation: page
 * "FlashAttention-3 ...", section "Analyse").  For each (b, h, block of 128 rows):
 * a = max|x|; scales[b,h,blk] = a/448; xq = cvt.rn.satfinite.e4m3(x * (448/a)), both
 * divisions correctly rounded fp32.  A block of zeros stores scale 1.
 *   x       device fp32 [B,H,S,D]            (read)
 *   xq      device e4m3 bytes [B,H,S,D]      (written)
 *   scales  device fp32 [B,H,ceil(S/128)]    (written)
 * D must be a multiple of 16 and at most 256.
 */
ATTN_API int attn_quantize_e4m3(const float* x, void* xq, float* scales, int B, int H, int S, int D,
                       void* stream);

/*
 * attn_fwd_fp8 — attention forward on e4m3 Q, K, V with per-128-row fp32 block scales
 * (as attn_quantize_e4m3 writes).  Scores use sQ*sK folded into the logit scale; P is
 * quantised to e4m3 before P.V with the V block scale folded in as sV[kt]/max_kt(sV);
 * the output is multiplied back by max_kt(sV).  Row sums use the unquantised P.
 *   q8, k8, v8   device e4m3 [B,H,S,D]; q_scale/k_scale/v_scale device fp32
 *   [B,H,ceil(S/128)]; o bf16 [B,H,Sq,D]; lse fp32 [B,H,Sq].
 * Other arguments as attn_fwd (D = 128 only).
 */
ATTN_API int attn_fwd_fp8(const void* q8, const void* k8, const void* v8,
                 const float* q_scale, const float* k_scale, const float* v_scale,
                 void* o, float* lse,
                 int B, int H, int Sq, int Sk, int D, float scale,
                 int mask_kind, int window, float softcap,
                 const float* alibi_slopes, const int* doc_ids, void* stream);

/*
 * attn_quantize_mxfp4 — MXFP4 quantiser for the FP4 forward (page "Hardware-Aware FP4
 * FlashAttention-4", summary paragraph: the forward runs on the FP4 tensor cores).  Element
 * format e2m1; one power-of-two scale per 32 consecutive elements of the contraction axis,
 * stored as the E8M0 byte X + 127 with X = floor(log2 max|x|) - 2 (an all-zero block stores
 * 0); element = e2m1 round-to-nearest-even, saturating at 6, of x * 2^-X.
 *   x     device bf16 [B,H,S,D], D = 128 (read)
 *   transpose = 0 (Q, K): xq bytes [B,H,S,64] (element d in byte d/2, low nibble for even d);
 *       x_sf bytes [B,H,ceil(S/128),512] (written).
 *   transpose = 1 (V): xq bytes [B,H,128,Sp/2], Sp = S rounded up to 128 (row d holds the
 *       keys; keys >= S are zero); x_sf bytes [B,H,Sp/128,512] (written).
 * Scale atom layout (what the tensor core reads, 128 rows x 4 blocks per 512 bytes): the
 * scale of row r (0..127 within the atom) and block k (0..3) is byte 16*(r%32) + 4*(r/32) + k.
 * Rows of the last atom past S get scale byte 0.  Pointers 16-byte aligned.  Returns
 * ATTN_ERR_INVALID for a bad argument (nothing launched).
 */
ATTN_API int attn_quantize_mxfp4(const void* x, void* xq, void* x_sf, int B, int H, int S, int D,
                                 int transpose, void* stream);

/*
 * attn_fwd_fp4 — attention forward for non-causal inference on MXFP4 Q, K, V with Direct-P
 * (page "Hardware-Aware FP4 FlashAttention-4", Direct-P paragraphs: the scores are mapped
 * straight to the FP4 codes the tensor cores multiply).  Both products run on the FP4 tensor
 * cores.  P: for each row and block of 32 keys, E = floor(max t) - 2 with t = scale *
 * log2(e) * s; code = clip(rint(2 (t - E) + 2), 0, 7) (the score rounded to the nearest
 * half octave above 2^E), block scale 2^E.  O = sum P~ v / sum P~ and LSE = ln(sum P~), P~
 * the e2m1 magnitudes times the block scales.  No mask (all keys < Sk visible).
 *   q4 [B,H,Sq,64], k4 [B,H_kv,Sk,64], vt4 [B,H_kv,128,Sp/2] and their scale atoms, as
 *   attn_quantize_mxfp4 writes them (D = 128); o bf16 [B,H,Sq,128]; lse fp32 [B,H,Sq].
 * H must be a multiple of H_kv (query head h reads key/value head h / (H/H_kv)).  Device
 * pointers, 16-byte aligned, caller-owned; nothing is allocated.  Errors as attn_fwd.
 */
ATTN_API int attn_fwd_fp4(const void* q4, const void* k4, const void* vt4, const void* q_sf,
                          const void* k_sf, const void* v_sf, void* o, float* lse, int B, int H,
                          int H_kv, int Sq, int Sk, float scale, void* stream);

/*
 * attn_get_status — synchronises `stream`, then returns and clears the current device's
 * status word: ATTN_OK, or ATTN_ERR_TIMEOUT if a kernel's bounded wait ran out since the
 * last call (that kernel abandoned its work item and left its outputs undefined),
 * ATTN_ERR_INVALID if attn_fwd_varlen met sequence offsets outside its tensors, or
 * ATTN_ERR_CUDA if the synchronisation itself failed.
 */
ATTN_API int attn_get_status(void* stream);

/* attn_strerror — static description of a status code (never NULL). */
ATTN_API const char* attn_strerror(int code);

/*
 * attn_shutdown — releases host-side caches and returns the current device's pooled
 * stream-ordered workspace memory to the system.  Safe to call more than once.
 */
ATTN_API void attn_shutdown(void);

/*
 * attn_debug_set_fault — test hook for the bounded waits.  A nonzero value makes the
 * next attention launches skip one producer signal inside the kernel, so that the
 * consumer's bounded wait runs out (about `timeout_ms` milliseconds) and the kernel
 * records ATTN_ERR_TIMEOUT and returns.  0 restores normal operation.  Never set it in
 * production.
 */
ATTN_API void attn_debug_set_fault(int skip_signal, int timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
