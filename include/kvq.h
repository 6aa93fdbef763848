/*
 * kvq.h -- C ABI of libkvq: blockwise NVFP4 quantization of attention K/V caches on
 * NVIDIA B200 (sm_100a), and dequantization back to bf16.
 *
 * Format (the pages' method, restated):
 *   - A tensor is a flat array of bf16 rows of head_dim elements. Every 16 consecutive
 *     elements of a row form a block.
 *   - Each element is stored as an FP4 e2m1 code (sign, 2 exponent bits, 1 mantissa
 *     bit; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), two codes per byte, the even element
 *     in the low nibble ("How NVFP4 Quantization Works in LongLive 2.0 for Transformer
 *     Inference", section "Stage 1: Weight Quantization", step 3).
 *   - Each block has one FP8 e4m3 scale byte ("Understanding the NVFP4 Format and
 *     Architecture": block scales quantized to FP8).
 *   - Each tensor (or each appended chunk of a cache) has one fp32 amax. Its global
 *     scale is gs = amax / (6 * 448) ("Stage 3: KV-Cache De-quantization at
 *     Inference", step 3).
 *
 * Quantization of one block, with amax_b = max |x| over the block and a denominator
 * R (6 for static_6, 4 for static_4; rule mse tries both):
 *     c   = e4m3_rne_satfinite((amax_b / R) / gs)        (c = 0 when gs == 0)
 *     S   = e4m3_value(c) * gs
 *     inv = 1 / S, replaced by 0 when it is infinite
 *     q_i = e2m1_rne_satfinite(x_i * inv)                 (sign kept, also for zero)
 *   Rule mse keeps R = 4 only when its squared error is strictly smaller. The error is
 *   the sum of (x_i - value(q_i) * S)^2, each residual one fused multiply-add, the squares
 *   accumulated by fused multiply-add into an even-position and an odd-position partial
 *   sum (index order), which are then added. All arithmetic is IEEE fp32,
 *   round-to-nearest-even. ("How to Use KV Cache Quantization with LongLive's
 *   LongLiveQuantizationConfig", section "Configuration Parameters Reference": scale
 *   rules static_6, static_4 and mse.)
 * Dequantization: y_i = bf16_rne(value(q_i) * S), the product rounded to fp32 first
 * ("CUDA De-quantization Pipeline"; "Stage 3", steps 2-3).
 *
 * Conventions for every call:
 *   - Pointers named "device" are CUDA device (or managed) memory that the caller
 *     allocates, owns and frees. The library never allocates or frees memory and keeps
 *     no state between calls, with two stated exceptions: kvq_attention_noalloc's
 *     built-in scratch array (see there) and the per-device error word that
 *     kvq_device_status reads. Host pointers are read before the call returns.
 *   - Work is queued on `stream` (a cudaStream_t; NULL is the legacy default stream)
 *     and runs asynchronously; results are valid once the stream has been
 *     synchronized. Calls on the same stream run in order.
 *   - Arguments are checked on the host before anything is queued. On any error
 *     nothing is launched and the outputs are untouched (except KVQ_ERR_CUDA, which is
 *     returned when a launch itself fails). kvq_last_error() describes the last
 *     failure of the calling thread.
 *   - Inputs must be finite bf16 (NaN or Inf give unspecified codes). n_elems == 0
 *     is a valid no-op.
 *   - Alignment: bf16 tensors (x, y) 32-byte aligned; packed codes 8-byte aligned.
 *     A misaligned pointer returns KVQ_ERR_MISALIGNED.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without including CUDA headers. */
typedef struct CUstream_st* kvq_stream_t;

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, unknown rule */
    KVQ_ERR_MISALIGNED = 2,  /* a pointer below the alignment stated above */
    KVQ_ERR_UNSUPPORTED = 3, /* a size beyond what the kernels index (see each call) */
    KVQ_ERR_CAPACITY = 4,    /* a cache range past capacity_rows */
    KVQ_ERR_CUDA = 5,        /* a CUDA runtime error while queuing work */
    KVQ_ERR_TIMEOUT = 6      /* a bounded wait inside a kernel gave up (kvq_device_status) */
} kvq_status;

/* Block-scale rule ("Configuration Parameters Reference": scale_rule). */
typedef enum {
    KVQ_RULE_STATIC_6 = 0, /* scale = amax_b / 6 */
    KVQ_RULE_STATIC_4 = 1, /* scale = amax_b / 4 */
    KVQ_RULE_MSE = 2       /* per block, the one of the two with the lower squared error */
} kvq_scale_rule;

/* Largest number of tensors one kvq_*_batch launch covers; larger batches are split
 * into several launches. */
#define KVQ_MAX_BATCH 64

/*
 * kvq_quantize -- quantize one bf16 tensor.
 *   Defined by "Stage 1: Weight Quantization (FP32 to NVFP4)" steps 1-4 (block amax,
 *   block scale by the rule, two FP4 values per uint8, a global amax for the tensor)
 *   and "FP4 Quantization in the Causal Model" (each K and V block quantized on its own).
 *   x        device, bf16[n_elems], 32-byte aligned. Read only.
 *   n_elems  number of elements, a multiple of head_dim (at most 2^36).
 *   head_dim row length, a positive multiple of 16.
 *   rule     KVQ_RULE_*.
 *   amax_in  device, 1 float, or NULL. When given, it is used as the tensor amax (the
 *            caller already knows it and the amax pass is skipped).
 *   amax_out device, 1 float, or NULL. Receives the amax used (the computed one, or a
 *            copy of *amax_in). At least one of amax_in / amax_out must be non-NULL.
 *   packed   device, uint8[n_elems / 2], 8-byte aligned. Written.
 *   scales   device, uint8[n_elems / 16] (e4m3 codes, one per block, same order). Written.
 * When the amax is computed for a batch of two or more tensors of up to 2^21 blocks (64
 * MiB of bf16) each (kvq_quantize_batch, kvq_append_batch), amax pass and quantization
 * run in one launch (otherwise in two): the tiles of the amax pass fold their
 * maxima into *amax_out, and the quantize tiles of the same launch wait for it there, so
 * the slot holds intermediate values until the stream reaches the end of the call. Such
 * a wait is bounded (2 s); if it gives up, the tensor's outputs are left unwritten,
 * *amax_out is set to NaN and kvq_device_status() reports KVQ_ERR_TIMEOUT. That only
 * happens when the launch cannot get its CTAs onto the GPU, e.g. another stream holds
 * every SM for longer than the bound.
 */
kvq_status kvq_quantize(const void* x, int64_t n_elems, int32_t head_dim, kvq_scale_rule rule,
                        const float* amax_in, float* amax_out, uint8_t* packed, uint8_t* scales,
                        kvq_stream_t stream);

/*
 * kvq_dequantize -- the inverse of kvq_quantize, to bf16 ("CUDA De-quantization
 *   Pipeline": packed cache + scale factors -> bf16; "Stage 3" steps 2-3).
 *   packed  device, uint8[n_elems / 2], 8-byte aligned.
 *   scales  device, uint8[n_elems / 16].
 *   amax    device, 1 float (the amax kvq_quantize wrote).
 *   y       device, bf16[n_elems], 32-byte aligned. Written; same element order as x.
 */
kvq_status kvq_dequantize(const uint8_t* packed, const uint8_t* scales, const float* amax, int64_t n_elems,
                          int32_t head_dim, void* y, kvq_stream_t stream);

/*
 * kvq_quantize_batch -- n_tensors independent kvq_quantize calls on tensors of the same
 *   n_elems and head_dim, in one set of launches (e.g. one layer's K and V). Each tensor
 *   has its own amax, exactly as if quantized alone.
 *   xs, packed, scales  host arrays of n_tensors device pointers (as in kvq_quantize).
 *   amax_in   host array of n_tensors device pointers, or NULL: compute every amax.
 *   amax_out  host array of n_tensors device pointers, or NULL when amax_in is given.
 *             When the amax is computed, every tensor needs its own slot (two tensors
 *             sharing one return KVQ_ERR_INVALID_ARG).
 *   At most KVQ_MAX_BATCH tensors share a launch; more are split.
 */
kvq_status kvq_quantize_batch(const void* const* xs, int32_t n_tensors, int64_t n_elems, int32_t head_dim,
                              kvq_scale_rule rule, const float* const* amax_in, float* const* amax_out,
                              uint8_t* const* packed, uint8_t* const* scales, kvq_stream_t stream);

/*
 * kvq_quantize_launches -- host only: the number of kernels kvq_quantize_batch (and
 *   kvq_append_batch, kvq_quantize_dequantize) launches for n_tensors tensors of n_elems
 *   elements: per group of KVQ_MAX_BATCH tensors, 1 when the amax is given (amax_given
 *   != 0), else 2 (a slot clear and the one-launch amax + quantize, for groups of two or
 *   more tensors of up to 2^21 blocks each) or 3 (clear, amax pass, quantize: a single
 *   tensor, or larger tensors). For 16-byte-aligned packed buffers; writes *launches (0
 *   for empty tensors).
 */
kvq_status kvq_quantize_launches(int32_t n_tensors, int64_t n_elems, int32_t head_dim, int32_t amax_given,
                                 int32_t* launches);

/*
 * kvq_dequantize_batch -- n_tensors independent kvq_dequantize calls of the same size in
 *   one set of launches. packed, scales, amax, ys: host arrays of n_tensors device pointers.
 */
kvq_status kvq_dequantize_batch(const uint8_t* const* packed, const uint8_t* const* scales,
                                const float* const* amax, int32_t n_tensors, int64_t n_elems, int32_t head_dim,
                                void* const* ys, kvq_stream_t stream);

/*
 * kvq_quantize_dequantize -- the fused round trip ("fake quantization", the
 *   static_blockwise_fp4_fake_quant of "How NVFP4 Quantization Works in LongLive 2.0",
 *   "Stage 1"): quantize x and write its bf16 reconstruction y in the same pass. y is
 *   bit-equal to kvq_quantize followed by kvq_dequantize.
 *   packed, scales  device outputs as in kvq_quantize, or both NULL to write only y.
 *   y               device, bf16[n_elems], 32-byte aligned. Written.
 *   Other arguments as in kvq_quantize.
 */
kvq_status kvq_quantize_dequantize(const void* x, int64_t n_elems, int32_t head_dim, kvq_scale_rule rule,
                                   const float* amax_in, float* amax_out, uint8_t* packed, uint8_t* scales,
                                   void* y, kvq_stream_t stream);

/*
 * A packed K or V cache of one layer, in device memory, token-major: row
 * t * heads + h holds head h of token t, head_dim elements. Rows are grouped in chunks
 * of rows_per_chunk (one chunk = the rows one append writes, e.g. one latent frame of
 * 1560 tokens x heads); every chunk has its own amax, written by the append that filled
 * it ("FP4 Quantization in the Causal Model": every new K/V block is quantized on its
 * own). kvq_cache_bytes gives the sizes.
 */
typedef struct {
    uint8_t* packed;        /* device, capacity_rows * head_dim / 2 bytes, 8-byte aligned */
    uint8_t* scales;        /* device, capacity_rows * head_dim / 16 bytes */
    float* amax;            /* device, ceil(capacity_rows / rows_per_chunk) floats */
    int64_t capacity_rows;  /* rows the cache holds */
    int64_t rows_per_chunk; /* rows per append chunk (> 0) */
    int32_t head_dim;       /* positive multiple of 16 */
} kvq_cache;

/*
 * kvq_append -- quantize-on-write: quantize n_rows new rows x into the cache at
 *   row_offset, with their own amax in cache->amax[row_offset / rows_per_chunk]
 *   ("KV Cache Quantization for Self-Forcing Video Generation", appendix Table 3:
 *   quantize-on-write every step, block size 16).
 *   cache      host pointer to the cache view.
 *   row_offset first row written; a multiple of rows_per_chunk.
 *   x          device, bf16[n_rows * head_dim], 32-byte aligned.
 *   n_rows     0 .. rows_per_chunk; row_offset + n_rows <= capacity_rows
 *              (else KVQ_ERR_CAPACITY).
 */
kvq_status kvq_append(const kvq_cache* cache, int64_t row_offset, const void* x, int64_t n_rows,
                      kvq_scale_rule rule, kvq_stream_t stream);

/*
 * kvq_append_batch -- n_tensors appends of the same n_rows in one set of launches
 *   (e.g. every layer's K and V of one frame).
 *   caches      host array of n_tensors cache views (same head_dim).
 *   row_offsets host array of n_tensors row offsets (each a multiple of its
 *               rows_per_chunk).
 *   xs          host array of n_tensors device pointers, bf16[n_rows * head_dim] each.
 *   The tensors must not overlap one another.
 */
kvq_status kvq_append_batch(const kvq_cache* caches, const int64_t* row_offsets, const void* const* xs,
                            int32_t n_tensors, int64_t n_rows, kvq_scale_rule rule, kvq_stream_t stream);

/*
 * kvq_dequantize_cache -- dequantize cache rows [row_begin, row_end) to bf16, each row
 *   with the amax of its chunk ("Stage 3: KV-Cache De-quantization at Inference";
 *   Self-Forcing study, appendix Table 3: the active cache goes back to dense BF16
 *   before attention).
 *   y  device, bf16[(row_end - row_begin) * head_dim], 32-byte aligned. Written.
 *   row_end <= capacity_rows (else KVQ_ERR_CAPACITY).
 */
kvq_status kvq_dequantize_cache(const kvq_cache* cache, int64_t row_begin, int64_t row_end, void* y,
                                kvq_stream_t stream);

/*
 * kvq_dequantize_cache_batch -- the same row range of n_tensors caches (same head_dim)
 *   into n_tensors outputs, in one set of launches.
 *   ys  host array of n_tensors device pointers.
 */
kvq_status kvq_dequantize_cache_batch(const kvq_cache* caches, void* const* ys, int32_t n_tensors,
                                      int64_t row_begin, int64_t row_end, kvq_stream_t stream);

/*
 * kvq_attention -- softmax attention out = softmax(softmax_scale * Q K^T) V per head,
 *   reading K and V straight from their NVFP4 caches: each tile of keys is dequantized
 *   in on-chip memory to the same bf16 values kvq_dequantize_cache writes, so no dense
 *   bf16 copy of the cache is ever stored ("How to Use KV Cache Quantization with
 *   LongLive's LongLiveQuantizationConfig", "CUDA De-quantization Pipeline": the cache
 *   is dequantized while attention runs; Self-Forcing study, abstract and Figure 6: the
 *   transient BF16 buffers of dequantize-then-attend set the peak memory). Every query
 *   attends to cache tokens [0, n_keys) (no mask); P is rounded to bf16 before P V and
 *   both products accumulate in fp32 on the tensor cores.
 *   q            device, bf16[n_queries, heads, 128] (token-major), 16-byte aligned.
 *   k_cache,     host pointers to the K and V cache views: rows are token * heads + head,
 *   v_cache      head_dim 128, rows_per_chunk a multiple of heads and equal in both,
 *                n_keys * heads <= capacity_rows (else KVQ_ERR_CAPACITY); packed 16-byte,
 *                scales 8-byte aligned; head_dim other than 128 is KVQ_ERR_UNSUPPORTED.
 *   n_keys       >= 1 cached tokens to attend to.
 *   softmax_scale  positive and finite (e.g. 1/sqrt(128)).
 *   out          device, bf16[n_queries, heads, 128], 16-byte aligned. Written.
 *   workspace    device scratch for the partial results of key splits, 16-byte aligned,
 *                workspace_bytes long; may be NULL with 0 bytes. The call splits the keys
 *                over more work units (to fill the GPU) only as far as the workspace
 *                holds their partials; kvq_attention_workspace_bytes gives the size that
 *                allows the split it would choose on the current device.
 *   status       device int, set to 1 if an on-chip wait timed out (the output is then
 *                incomplete); never cleared by the call.
 * kvq_attention_workspace_bytes -- host only: that size for these sizes (0 when no split
 *   would be used).
 * kvq_attention_launches -- host only: how many kernels one kvq_attention call of these
 *   sizes launches on the current device when given that workspace (1 to 4: the query
 *   rows run in one or two parts, on CTA pairs or single CTAs, each followed by a
 *   combine kernel when it splits its keys); 0 for n_queries == 0.
 */
kvq_status kvq_attention(const void* q, int32_t n_queries, int32_t heads, const kvq_cache* k_cache,
                         const kvq_cache* v_cache, int64_t n_keys, float softmax_scale, void* out, void* workspace,
                         uint64_t workspace_bytes, int* status, kvq_stream_t stream);
kvq_status kvq_attention_workspace_bytes(int32_t n_queries, int32_t heads, int64_t n_keys, uint64_t* bytes);
kvq_status kvq_attention_launches(int32_t n_queries, int32_t heads, int64_t n_keys, int32_t* launches);

/*
 * kvq_attention_noalloc -- kvq_attention without a workspace argument, for callers that
 *   cannot allocate device memory: code running inside a host framework that owns the
 *   GPU's memory through its own pool and budget (a cudaMalloc there would bypass its
 *   accounting or fail under its limit), or a latency-critical loop that cannot afford
 *   cudaMalloc's implicit device synchronization. It allocates nothing: the partial
 *   results of the key split live in a 32 MiB array built into the library, which every
 *   GPU that runs the attention kernels holds until the process exits. (The pages have
 *   no counterpart; this is a deployment convenience of this library.)
 *   Arguments, result and errors are those of kvq_attention, plus:
 *   - sizes whose key split needs more than 32 MiB (kvq_attention_workspace_bytes above
 *     32 MiB) return KVQ_ERR_CAPACITY with the needed size in kvq_last_error();
 *   - every call looks up the array's device address on the current device (a host-side
 *     query that allocates nothing; the first one on a device may load the library's
 *     device code, so make the first call before any stream capture);
 *   - every call on a GPU shares the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race on it and must be ordered by the caller. Nothing
 *     in it needs to start at zero: a call whose *status stays 0 writes every partial it
 *     reads; after a wait that gave up (*status 1) out may hold an earlier call's data.
 */
kvq_status kvq_attention_noalloc(const void* q, int32_t n_queries, int32_t heads, const kvq_cache* k_cache,
                                 const kvq_cache* v_cache, int64_t n_keys, float softmax_scale, void* out,
                                 int* status, kvq_stream_t stream);

/*
 * RTN integer codecs: the RTN_INT4 / RTN_INT2 rows of "KV Cache Quantization for
 * Self-Forcing Video Generation: A 33-Method Empirical Study", appendix Table 3
 * (symmetric blockwise quantization of K and V, block_size=16, 4-bit / 2-bit packed
 * storage plus per-block scales); RTN_K2_V4 is bits = 2 for K and 4 for V. Per block of
 * 16 elements, qmax = 2^(bits-1) - 1:
 *     S = bf16_rne(amax_b / qmax)            one bf16 scale per block (16 bits per 16
 *                                            values: the study's 5.33x for INT2)
 *     q = round_half_even(x / S) in [-qmax, qmax], 0 when S == 0 (IEEE fp32 quotient)
 *     y = bf16_rne(q * S)
 * Codes are two's complement; INT4 two per byte (even element in the low nibble), INT2
 * four per byte (element 4j + k in bits 2k..2k+1). There is no global scale. A cache
 * append or range read is the same call on pointers offset into the cache buffers.
 *
 * kvq_rtn_quantize
 *   x        device, bf16[n_elems], 32-byte aligned (n_elems a multiple of head_dim).
 *   bits     2 or 4.
 *   packed   device, uint8[n_elems * bits / 8], 2*bits-byte aligned. Written.
 *   scales   device, bf16 bit patterns uint16[n_elems / 16], 2-byte aligned. Written.
 * kvq_rtn_dequantize -- the inverse; y device bf16[n_elems], 32-byte aligned. Written.
 * The _batch forms take host arrays of n_tensors device pointers of one size and bits.
 */
kvq_status kvq_rtn_quantize(const void* x, int64_t n_elems, int32_t head_dim, int32_t bits, uint8_t* packed,
                            uint16_t* scales, kvq_stream_t stream);
kvq_status kvq_rtn_dequantize(const uint8_t* packed, const uint16_t* scales, int64_t n_elems, int32_t head_dim,
                              int32_t bits, void* y, kvq_stream_t stream);
kvq_status kvq_rtn_quantize_batch(const void* const* xs, int32_t n_tensors, int64_t n_elems, int32_t head_dim,
                                  int32_t bits, uint8_t* const* packed, uint16_t* const* scales,
                                  kvq_stream_t stream);
kvq_status kvq_rtn_dequantize_batch(const uint8_t* const* packed, const uint16_t* const* scales, int32_t n_tensors,
                                    int64_t n_elems, int32_t head_dim, int32_t bits, void* const* ys,
                                    kvq_stream_t stream);

/*
 * RECENT cache policy: the RTN_INT4 RECENT2 method of "KV Cache Quantization for
 * Self-Forcing Video Generation" (appendix Table 3): the newest `recent_blocks` (2)
 * frame-blocks of a K or V cache are kept in bf16 ("recent_k / recent_v" state) and only
 * older blocks are RTN-quantized; a read dequantizes the quantized prefix and copies the
 * bf16 tail back in. A frame-block is rows_per_block rows (tokens x heads) of head_dim.
 *   packed   device, RTN codes of capacity_blocks blocks: capacity_blocks * rows_per_block
 *            * head_dim * bits / 8 bytes (block b at offset b * its size), 2*bits-aligned.
 *   scales   device, bf16 scales, one per 16 elements, same block order, 2-byte aligned.
 *   recent   device, bf16 ring of recent_blocks blocks (block b in slot b % recent_blocks),
 *            32-byte aligned.
 * head_dim is a positive multiple of 16 with rows_per_block * head_dim a multiple of 16;
 * bits is 4 (the study's RECENT2 prefix) or 2.
 */
typedef struct {
    uint8_t* packed;
    uint16_t* scales;
    void* recent;
    int64_t capacity_blocks;
    int64_t rows_per_block;
    int32_t head_dim;
    int32_t bits;
    int32_t recent_blocks;
} kvq_recent_cache;

/*
 * kvq_recent_append_batch -- quantize-on-write of frame-block `block` into n_caches
 *   caches (e.g. every layer's K and V), blocks appended in order 0, 1, 2, ...: the
 *   block leaving the bf16 window (block - recent_blocks, if block >= recent_blocks) is
 *   RTN-quantized from its ring slot into the prefix, then x takes that slot.
 *   caches  host array of n_caches cache views (same rows_per_block, head_dim, bits,
 *           recent_blocks).
 *   xs      host array of n_caches device pointers, bf16[rows_per_block * head_dim] each,
 *           32-byte aligned.
 *   block < capacity_blocks, else KVQ_ERR_CAPACITY.
 */
kvq_status kvq_recent_append_batch(const kvq_recent_cache* caches, int32_t n_caches, int64_t block,
                                   const void* const* xs, kvq_stream_t stream);

/*
 * kvq_recent_read_batch -- the whole active cache of n_caches caches as bf16, n_blocks
 *   being the number of blocks appended so far (not checked; at most capacity_blocks,
 *   else KVQ_ERR_CAPACITY): blocks [0, n_blocks - r) dequantized from the prefix,
 *   r = min(recent_blocks, n_blocks), then the r newest blocks copied from the ring.
 *   ys  host array of n_caches device pointers, bf16[n_blocks * rows_per_block *
 *       head_dim] each, 32-byte aligned. Written.
 */
kvq_status kvq_recent_read_batch(const kvq_recent_cache* caches, int32_t n_caches, int64_t n_blocks,
                                 void* const* ys, kvq_stream_t stream);

/*
 * Blocked scale layout: the 128 x 4 tiles block-scaled MMA operands read ("How NVFP4
 * Quantization Works in LongLive 2.0", "Stage 3", step 1: the dequantizer first undoes
 * it, "from_blocked"). A [rows, cols] matrix of one-byte scales (row-major: the scales
 * array of kvq_quantize for a rows x head_dim tensor, cols = head_dim / 16) is padded
 * with zeros to rows' = ceil(rows/128)*128 and cols' = ceil(cols/4)*4 and cut into
 * 128 x 4 tiles of 512 bytes, in row-tile-major order; inside a tile, scale (r, c) sits
 * at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.
 *
 * kvq_scales_to_blocked    scales (device, rows*cols bytes) -> blocked (device,
 *                          kvq_blocked_scale_bytes bytes, 16-byte aligned, padding zeroed).
 * kvq_scales_from_blocked  the inverse (blocked 16-byte aligned); writes rows*cols bytes.
 * A blocked buffer that is not 16-byte aligned returns KVQ_ERR_MISALIGNED; the plain
 * scales have no alignment requirement.
 * kvq_blocked_scale_bytes  host only: rows' * cols'.
 */
kvq_status kvq_scales_to_blocked(const uint8_t* scales, int64_t rows, int32_t cols, uint8_t* blocked,
                                 kvq_stream_t stream);
kvq_status kvq_scales_from_blocked(const uint8_t* blocked, int64_t rows, int32_t cols, uint8_t* scales,
                                   kvq_stream_t stream);
kvq_status kvq_blocked_scale_bytes(int64_t rows, int32_t cols, uint64_t* bytes);

/*
 * kvq_cache_bytes -- host only. Bytes of a cache of `layers` layers x {K, V}, each
 *   capacity_tokens x heads rows of head_dim, chunks of tokens_per_chunk tokens:
 *     packed = 2*layers * capacity_tokens*heads*head_dim / 2
 *     scales = 2*layers * capacity_tokens*heads*head_dim / 16
 *     amax   = 2*layers * ceil(capacity_tokens / tokens_per_chunk) * 4
 *   (4.5 bits per element plus one float per chunk: "How NVFP4 Quantization Works",
 *   FAQ on memory savings; Self-Forcing study, Figure 6, compressed versus
 *   BF16-equivalent footprint). Any output pointer may be NULL.
 */
kvq_status kvq_cache_bytes(int32_t layers, int32_t heads, int64_t capacity_tokens, int32_t head_dim,
                           int64_t tokens_per_chunk, uint64_t* packed_bytes, uint64_t* scale_bytes,
                           uint64_t* amax_bytes);

/* Human-readable name of a status code (static string). */
const char* kvq_status_string(kvq_status status);

/* Description of the last error returned to the calling thread ("" if none). */
const char* kvq_last_error(void);

/* Library version, e.g. "0.1.0". */
const char* kvq_version(void);

/*
 * kvq_device_status -- errors that kernels of this library raised on the current device
 *   since the last clearing call: KVQ_ERR_TIMEOUT when a bounded wait inside a kernel gave
 *   up (see kvq_quantize), else KVQ_OK. The word is sticky and per device; clear != 0
 *   resets it. This call copies from the device, so it waits for the device's preceding
 *   work on the legacy default stream (and, with that stream's usual semantics, for the
 *   work it synchronizes with); call it after synchronizing the streams of interest.
 *   Returns KVQ_ERR_CUDA if the copy fails. kvq_attention reports its own timeouts
 *   through its status argument instead.
 */
kvq_status kvq_device_status(int32_t clear);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
