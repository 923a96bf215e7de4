/*
 * thrift.h -- C ABI of the selective mixed-precision (FP16 / NVFP4) block
 * attention library for NVIDIA B200 (sm_100a).
 *
 * The method (page "ThriftAttention: Selective Mixed Precision for
 * Long-Context FP4 Attention", abstract; same page's summary, "technical
 * approach" items 2-5) computes prefill attention in two stages:
 *   1. a cheap heuristic picks a small fraction rho of (query block, key
 *      block) pairs to run in FP16                 -> thrift_select_blocks
 *   2. the picked pairs run in FP16, all other pairs in block-scaled FP4, and
 *      one online softmax merges both into one output -> thrift_attention
 * The FP4 operands come from                       -> thrift_quantize_nvfp4
 * and thrift_attention_fused chains all of them.
 *
 * Readings of points the pages leave open (each is fixed, not tunable):
 *   - NVFP4: E2M1 codes with one E4M3 scale per 16 consecutive elements along
 *     the contracted axis, scale = E4M3_rn(amax/6) with amax/6 rounded to
 *     FP32, code = E2M1_rn(x/scale) (ties to even, saturating, sign kept);
 *     a zero scale encodes the whole group as +0.
 *   - Q and K are quantised along D, V along the key axis, P (the softmax
 *     numerators) per 16 keys, at a fixed pre-scale of 2^11 that the output
 *     divides out again.
 *   - Heuristic: score(i,j) = fl32(sm_scale * fl32(mean_q(i) . mean_k(j)))
 *     from FP32 block means; per (batch, query head) keep
 *     k = ceil(rho * #valid_pairs - 1e-9) pairs, diagonal pairs (i,i) and
 *     key-block-0 pairs (i,0) first, then by score, ties to the lower linear
 *     index i*nb + j.
 *   - Online softmax keeps an integer running maximum of the log2-domain
 *     logits, so every rescale is an exact power of two; the row sum l adds
 *     the unquantised P.
 *
 * Conventions for every call:
 *   - Pointers named Q, K, V, O, mask, codes, scales, ws are DEVICE pointers,
 *     owned by the caller; the library allocates no device memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); calls only
 *     enqueue work and return without synchronising.
 *   - Arguments are validated on the host before any launch; on error nothing
 *     is launched and the status says why.
 *   - Device-side faults are never raised on purpose: every wait inside a
 *     kernel is bounded; a timeout sets a device error word that
 *     thrift_last_device_error() reads (and clears).
 *   - Tensors are contiguous, row-major:
 *       Q [B][Hq][N][D] fp16, K and V [B][Hkv][N][D] fp16, O like Q.
 *     Query head h reads key/value head h / (Hq/Hkv).
 *   - Supported shapes: D in {64, 128}; blk in {64, 128}; N a positive
 *     multiple of blk; Hq a multiple of Hkv; all sizes positive.  Other
 *     shapes return THRIFT_ERR_UNSUPPORTED.
 */
#ifndef THRIFT_H_
#define THRIFT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define THRIFT_API __attribute__((visibility("default")))
#else
#define THRIFT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  THRIFT_OK = 0,
  THRIFT_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, rho outside [0,1] */
  THRIFT_ERR_UNSUPPORTED = 2, /* valid but unsupported shape (see above) */
  THRIFT_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch, attribute, copy) */
  THRIFT_ERR_TIMEOUT = 4,     /* a kernel gave up a bounded wait (device error word) */
  THRIFT_ERR_WORKSPACE = 5    /* workspace pointer null or too small */
} thrift_status;

typedef enum { THRIFT_Q = 0, THRIFT_K = 1, THRIFT_V = 2 } thrift_operand;

/* Problem shape.  sm_scale > 0 multiplies Q K^T (usually 1/sqrt(D)); causal = 1
 * masks key > query.  blk is the selection block (square, blk x blk). */
typedef struct {
  int B, Hq, Hkv, N, D, blk, causal;
  float sm_scale;
} thrift_shape;

/* Sizes of the NVFP4 copy of one operand.
 * Codes (canonical, also what the attention kernel reads by TMA):
 *   Q/K: [B][H][N][D/2] bytes, element d in the low nibble of byte d/2 when
 *        d is even, high nibble when odd;
 *   V:   [B][Hkv][D][N/2] bytes (keys contiguous), key n in nibble n%2.
 * Scales (E4M3 bytes) in the tensor-core scale-factor layout, with
 * NT = ceil(N/128):
 *   Q/K: [B][H][NT][D/64][32][4][4]; the scale of row n, group g = d/16 sits at
 *        ((bh*NT + n/128)*(D/64) + g/4)*512 + (n%32)*16 + ((n%128)/32)*4 + g%4;
 *   V:   [B][Hkv][2*NT][32][4][4]; the scale of channel d, key group n/16 sits at
 *        (bh*2*NT + n/64)*512 + (d%32)*16 + (d/32)*4 + (n%64)/16.
 * Padding bytes (rows past N, channels past D) are written as 0.
 * Returns INVALID_ARG / UNSUPPORTED like the calls below. */
THRIFT_API thrift_status thrift_quant_bytes(const thrift_shape* shape, thrift_operand op, size_t* codes_bytes,
                                 size_t* scales_bytes);

/* NVFP4 quantisation of one operand (Q or K along D, V along keys).
 * x: fp16 device tensor of the operand's shape; codes/scales: device buffers
 * of thrift_quant_bytes() sizes.  Block-scaled FP4 as the pages' prior work
 * on Blackwell ("ThriftAttention" abstract); the format is the NVFP4 reading
 * above. */
THRIFT_API thrift_status thrift_quantize_nvfp4(const void* x, thrift_operand op, const thrift_shape* shape, void* codes,
                                    void* scales, void* stream);

/* Q or K quantised as thrift_quantize_nvfp4 does (identical codes and scales)
 * and pooled in the same pass, so the fp16 tensor is read from HBM once:
 * means [B][H][N/blk][D] FP32 receives the block means of the selection
 * heuristic (ThriftAttention abstract: the cheap heuristic that picks the
 * block pairs), each the FP64 sum of a block's blk rows divided by blk,
 * rounded once to FP32, identical to what thrift_select_blocks computes
 * internally.  op: THRIFT_Q (H = Hq) or THRIFT_K (H = Hkv); means 4-byte
 * aligned.  Feed the means to thrift_select_blocks_pooled.  Errors as for
 * thrift_quantize_nvfp4; INVALID_ARG for op V. */
THRIFT_API thrift_status thrift_quantize_pool_nvfp4(const void* x, thrift_operand op, const thrift_shape* shape,
                                                    void* codes, void* scales, float* means, void* stream);

/* MXFP8 copies for 8-bit block pairs (mask value 3 of the tiered selection),
 * after TriAttention's 8-bit precision (abstract on the paper page of arXiv
 * 2611.07256): the OCP microscaling format with E4M3 elements and one E8M0
 * scale per 32 consecutive elements, X = 2^(floor(log2 amax) - 8); element =
 * E4M3(v / X), nearest even, saturating at 448; an all-zero group has scale
 * byte 0 and zero codes.  Q, K along D, V along keys.
 * Codes: Q/K [B][H][N][D] bytes; V [B][Hkv][D][N] bytes (keys contiguous).
 * Scales, NT = ceil(N/128), one 512-byte chunk per 128-row tile:
 *   Q/K: byte (bh*NT + n/128)*512 + (n%32)*16 + ((n%128)/32)*4 + d/32;
 *   V:   byte (bh*NT + n/128)*512 + (d%32)*16 + (d/32)*4 + (n%128)/32.
 * Bytes no element maps to are 0.  Errors as for thrift_quantize_nvfp4. */
THRIFT_API thrift_status thrift_quant8_bytes(const thrift_shape* shape, thrift_operand op, size_t* codes_bytes,
                                             size_t* scales_bytes);
THRIFT_API thrift_status thrift_quantize_mxfp8(const void* x, thrift_operand op, const thrift_shape* shape,
                                               void* codes, void* scales, void* stream);

/* Workspace bytes thrift_select_blocks and thrift_select_blocks_vertical_window
 * need (block means, pooled scores, column ranks). */
THRIFT_API thrift_status thrift_select_workspace_bytes(const thrift_shape* shape, size_t* bytes);

/* Stage 1 (ThriftAttention abstract: a cheap heuristic picks the few
 * query-key block pairs that matter most): writes
 * mask [B][Hq][nb][nb] (nb = N/blk) with 1 for pairs computed in FP16 and 0
 * for FP4 pairs and for invalid (causal, j > i) pairs.
 * rho in [0,1]; ws: device workspace of at least
 * thrift_select_workspace_bytes() bytes (contents need not be initialised). */
THRIFT_API thrift_status thrift_select_blocks(const void* Q, const void* K, const thrift_shape* shape, double rho,
                                   uint8_t* mask, void* ws, size_t ws_bytes, void* stream);

/* thrift_select_blocks from precomputed block means (qm [B][Hq][nb][D],
 * km [B][Hkv][nb][D], FP32, as thrift_quantize_pool_nvfp4 writes them): the
 * same scores, budget and mask, without a pooling pass.  ws as for
 * thrift_select_blocks (the block-mean part of it is not used). */
THRIFT_API thrift_status thrift_select_blocks_pooled(const float* qm, const float* km, const thrift_shape* shape,
                                                     double rho, uint8_t* mask, void* ws, size_t ws_bytes,
                                                     void* stream);

/* Stage 1 with two more classes, 8-bit and skipped pairs, after
 * TriAttention's tile precisions (abstract on the paper page of arXiv
 * 2611.07256: interactions that matter least are skipped, the precision of
 * the rest lowered, 8-bit among the precisions).  The method's ranking (as
 * thrift_select_blocks) is cut in four per (batch, query head):
 *   the first k16 = ceil(rho * #valid - 1e-9) pairs          -> 1 (FP16)
 *   the next  k8  = min(ceil(rho8 * #valid - 1e-9),
 *                       #valid - k16) pairs                  -> 3 (MXFP8)
 *   the last  ks  = min(ceil(sigma * #valid - 1e-9),
 *                       #valid - max(k16 + k8, 2 nb - 1))    -> 2 (skipped)
 *   the others                                               -> 0 (NVFP4)
 * so the forced pairs (diagonal and key block 0, 2 nb - 1 of them), the FP16
 * and the 8-bit pairs are never skipped; rho8 = sigma = 0 gives
 * thrift_select_blocks' mask.  thrift_attention_tiered treats a skipped pair
 * as absent from the softmax.  rho, rho8, sigma in [0, 1]; workspace, layout
 * and errors as for thrift_select_blocks. */
THRIFT_API thrift_status thrift_select_blocks_tiered(const void* Q, const void* K, const thrift_shape* shape,
                                                     double rho, double rho8, double sigma, uint8_t* mask, void* ws,
                                                     size_t ws_bytes, void* stream);

/* An alternative stage 1 on the same FP16 budget, after HyQuant (abstract in
 * the body of the page titled "LampAttention: Look-Ahead Mixed-Precision
 * FlashAttention for Dedicated Accelerators"): HyQuant keeps full precision
 * for the keys that many queries attend to (vertical lines of the attention
 * map) and for a sliding window beside the diagonal, chosen by a cheap signal
 * of the attention pattern.  At block granularity, per (batch, query head):
 *   - pooled scores s(i,j) exactly as thrift_select_blocks computes them;
 *   - column signal v_j = sum over valid rows i of softmax_j'(s(i,j'))[j], the
 *     pooled attention mass key block j receives (FP32, fixed summation
 *     order: per row the maximum, then the sum of exp(s - max); per column
 *     the sum over i in increasing order); columns ranked by v descending,
 *     ties to the lower j;
 *   - the same budget k = ceil(rho * #valid_pairs - 1e-9); pairs ordered by
 *     (in the window: i - window < j <= i causal, |i - j| < window otherwise)
 *     first, then the column's rank, then s(i,j) descending, then lower i;
 *     the first k are kept.
 * window >= 0 in blocks (0: no window).  nb = N/blk must be <= 2048
 * (THRIFT_ERR_UNSUPPORTED otherwise).  Workspace, mask layout and errors as
 * for thrift_select_blocks; the workspace size is the same call. */
THRIFT_API thrift_status thrift_select_blocks_vertical_window(const void* Q, const void* K, const thrift_shape* shape,
                                                              double rho, int window, uint8_t* mask, void* ws,
                                                              size_t ws_bytes, void* stream);

/* thrift_select_blocks without a caller-supplied workspace.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory -- their GPU memory is owned by another allocator (a
 * framework's caching pool, a serving runtime that reserves the device at
 * start-up), or they are hooks called by a host program that gives them no
 * way to allocate.  It computes exactly what thrift_select_blocks computes,
 * with the same kernels, on a scratch array held in the library's own static
 * device memory:
 *   - the array is THRIFT_SELECT_STATIC_BYTES (16 MiB) per device, held by
 *     every GPU that loads the library until the process exits; shapes whose
 *     selection workspace (thrift_select_workspace_bytes) exceeds it return
 *     THRIFT_ERR_WORKSPACE;
 *   - it allocates nothing (no cudaMalloc, no cudaFree);
 *   - the first call on a device looks up the array's device address with
 *     that device current (a one-time set-up); make that first call before
 *     any stream capture;
 *   - every call shares the array and it keeps the last call's contents
 *     (nothing needs clearing: the kernels overwrite all they read); calls
 *     whose kernels overlap on the GPU, e.g. on two streams, race on it;
 *   - the looked-up address is kept for the life of the process, so a
 *     device reset (cudaDeviceReset) invalidates it, as it invalidates the
 *     device error word's (thrift_last_device_error): do not call the
 *     library on a device after resetting it.
 * Arguments and the mask output are as for thrift_select_blocks. */
#define THRIFT_SELECT_STATIC_BYTES ((size_t)16 << 20)
THRIFT_API thrift_status thrift_select_blocks_static(const void* Q, const void* K, const thrift_shape* shape,
                                                     double rho, uint8_t* mask, void* stream);

/* Stage 2 (ThriftAttention abstract: picked pairs in FP16, the others in
 * FP4, one online softmax merging both): O [B][Hq][N][D] fp16.
 * mask: as written by thrift_select_blocks (1 FP16, 0 NVFP4; any nonzero
 * byte counts as FP16, so masks with skipped or 8-bit pairs go to
 * thrift_attention_tiered instead); q4/qs, k4/ks, v4/vs: the NVFP4
 * copies written by thrift_quantize_nvfp4 for Q, K and V. */
THRIFT_API thrift_status thrift_attention(const void* Q, const void* K, const void* V, const uint8_t* mask, const void* q4,
                               const void* qs, const void* k4, const void* ks, const void* v4, const void* vs,
                               const thrift_shape* shape, void* O, void* stream);

/* thrift_attention for masks that may also hold 2 and 3, as written by
 * thrift_select_blocks_tiered.  A skipped pair (2) is absent from the softmax
 * (every query row must keep at least one key; the tiered selection never
 * skips the diagonal).  With blk = 128 the skipped key tiles are left out of
 * the kernel's work; with blk = 64 a skipped block inside a 128-key tile is
 * computed and masked.  An 8-bit pair (3) takes S from the MXFP8 copies of Q
 * and K, encodes P * 2^11 as MXFP8 per aligned group of 32 keys (E8M0 scale
 * 2^(floor(log2 amax) - 8) of the group's maximum, E4M3 codes; a group whose
 * scale byte would be 0 is encoded as zeros) and multiplies it with the
 * MXFP8 copy of V.
 *   q8, qs8, k8, ks8, v8, vs8: the MXFP8 copies from thrift_quantize_mxfp8
 *     (Q with THRIFT_Q, K with THRIFT_K, V with THRIFT_V), all six or none
 *     (THRIFT_ERR_INVALID_ARG otherwise); with them blk must be 128
 *     (THRIFT_ERR_UNSUPPORTED otherwise).
 * A mask byte the call cannot compute (3 without the copies, above 3) makes
 * thrift_last_device_error() return THRIFT_ERR_INVALID_ARG; that tile is
 * then computed in NVFP4.  Other arguments and errors as for
 * thrift_attention. */
THRIFT_API thrift_status thrift_attention_tiered(const void* Q, const void* K, const void* V, const uint8_t* mask,
                                                 const void* q4, const void* qs, const void* k4, const void* ks,
                                                 const void* v4, const void* vs, const void* q8, const void* qs8,
                                                 const void* k8, const void* ks8, const void* v8, const void* vs8,
                                                 const thrift_shape* shape, void* O, void* stream);

/* Workspace bytes of thrift_attention_fused (NVFP4 copies, mask and the
 * selection workspace, each 256-byte aligned). */
THRIFT_API thrift_status thrift_fused_workspace_bytes(const thrift_shape* shape, size_t* bytes);

/* Both stages in one call: quantise Q, K, V, select with budget rho, attend.
 * ws: device workspace of thrift_fused_workspace_bytes() bytes. */
THRIFT_API thrift_status thrift_attention_fused(const void* Q, const void* K, const void* V, const thrift_shape* shape,
                                     double rho, void* O, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of thrift_attention_fused_tiered for a given 8-bit budget
 * (the NVFP4 copies, mask, selection workspace and, when rho8 > 0, the MXFP8
 * copies; each part 256-byte aligned). */
THRIFT_API thrift_status thrift_fused_tiered_workspace_bytes(const thrift_shape* shape, double rho8, size_t* bytes);

/* The tiered path in one call: quantise Q, K, V to NVFP4 (and, when rho8 > 0,
 * to MXFP8), select with thrift_select_blocks_tiered(rho, rho8, sigma), attend
 * with thrift_attention_tiered.  The result equals those calls made one by
 * one.  rho8 > 0 needs blk = 128 (THRIFT_ERR_UNSUPPORTED otherwise).
 * ws: device workspace of thrift_fused_tiered_workspace_bytes(shape, rho8). */
THRIFT_API thrift_status thrift_attention_fused_tiered(const void* Q, const void* K, const void* V,
                                                       const thrift_shape* shape, double rho, double rho8,
                                                       double sigma, void* O, void* ws, size_t ws_bytes,
                                                       void* stream);

/* ---- decode: one new query row per (batch, query head) ----------------------
 * One decode step over the caches that prefill leaves behind: the fp16 K and
 * V and their NVFP4 copies from thrift_quantize_nvfp4.  The ThriftAttention
 * pages describe prefill only; re-using the block-scaled FP4 K/V of prefill
 * as a decode cache follows TriAttention (abstract on the paper page of
 * arXiv 2611.07256).  Reading: the query row is its own query block and sits
 * after the N cached keys, seeing all of them.
 *   - shape: B, Hq, Hkv, D, blk, sm_scale as for prefill, N = cache length;
 *     causal is ignored.  Decode calls other than thrift_pool_keys need
 *     D = 128, blk = 128 and Hq / Hkv <= 16 (THRIFT_ERR_UNSUPPORTED).
 *   - q: [B][Hq][D] fp16; O: [B][Hq][D] fp16; K, V: [B][Hkv][N][D] fp16;
 *     k4/ks, v4/vs: thrift_quantize_nvfp4(K, THRIFT_K) and (V, THRIFT_V)
 *     for the same shape.
 *   - selection: score_j = fl32(sm_scale * fl32(q . kmean_j)) over the nb =
 *     N/blk key blocks, kmean_j the FP32 block means of thrift_pool_keys (the
 *     means of the prefill heuristic); k = ceil(rho * nb - 1e-9) blocks, the
 *     first (j = 0) and the last (j = nb - 1) first, then by score, ties to
 *     the lower j.
 *   - attention: selected blocks in FP16, the others in NVFP4 (q encoded
 *     along D like a row of Q), the prefill's online softmax (integer
 *     maximum, P pre-scaled by 2^11, l over the unquantised P). */

/* FP32 block means of K: km [B][Hkv][nb][D] (exact FP64 sums of the fp16
 * rows, divided by blk, rounded once).  Any supported prefill shape. */
THRIFT_API thrift_status thrift_pool_keys(const void* K, const thrift_shape* shape, float* km, void* stream);

/* Decode selection: mask [B][Hq][nb] (u8, 1 = FP16 block). */
THRIFT_API thrift_status thrift_decode_select(const void* q, const float* km, const thrift_shape* shape, double rho,
                                              uint8_t* mask, void* stream);

/* Workspace bytes of thrift_decode_attention and thrift_decode_step (the
 * mask of thrift_decode_step, per-chunk partial results of both passes, and
 * per (batch, kv head) the key tiles some query head keeps in FP16). */
THRIFT_API thrift_status thrift_decode_workspace_bytes(const thrift_shape* shape, size_t* bytes);

/* Decode attention with a given mask [B][Hq][nb] (1 = FP16 block). */
THRIFT_API thrift_status thrift_decode_attention(const void* q, const void* K, const void* V, const void* k4,
                                                 const void* ks, const void* v4, const void* vs, const uint8_t* mask,
                                                 const thrift_shape* shape, void* O, void* ws, size_t ws_bytes,
                                                 void* stream);

/* Selection and attention in one call (km from thrift_pool_keys). */
THRIFT_API thrift_status thrift_decode_step(const void* q, const void* K, const void* V, const void* k4,
                                            const void* ks, const void* v4, const void* vs, const float* km,
                                            const thrift_shape* shape, double rho, void* O, void* ws,
                                            size_t ws_bytes, void* stream);

/* Synchronise `stream`, read and clear the device error word of the current
 * device: THRIFT_OK; THRIFT_ERR_TIMEOUT if a kernel gave up a bounded wait
 * since the last call; THRIFT_ERR_INVALID_ARG if a kernel met a mask byte it
 * cannot compute; THRIFT_ERR_CUDA if the synchronisation failed.  The word
 * keeps the first error recorded. */
THRIFT_API thrift_status thrift_last_device_error(void* stream);

/* Bound, in nanoseconds, of every wait inside the prefill attention kernels
 * (thrift_attention, thrift_attention_tiered and the fused entries) launched
 * after this call, process-wide; 2 s by default.  A kernel whose wait runs
 * out records THRIFT_ERR_TIMEOUT in the device error word
 * (thrift_last_device_error), raises an abort flag that makes every role of
 * its CTA leave its loop, drains its copies and tensor-core work, and
 * returns; the output of that launch is not written.  A shorter bound makes
 * failure detection faster; it must stay well above a kernel's longest
 * legitimate wait (microseconds on the supported shapes).  Returns
 * THRIFT_ERR_INVALID_ARG outside [1 us, 60 s]. */
THRIFT_API thrift_status thrift_set_wait_limit(uint64_t ns);

/* Static, human-readable name of a status. */
THRIFT_API const char* thrift_strerror(thrift_status status);

#ifdef __cplusplus
}
#endif

#endif /* THRIFT_H_ */
