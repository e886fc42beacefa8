/*
 * sage.h -- C ABI of the B200 (sm_100a) 8-bit quantized attention library
 * (libsage_b200.so).
 *
 * The operation is the forward pass of SageAttention as its article states it
 * ("SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
 * Acceleration", method section):
 *   1. K smoothing: K <- K - mean(K), the mean taken over the token axis, one
 *      value per channel (softmax(QK^T) = softmax(Q(K - mean K)^T));
 *   2. per-block INT8 quantization of Q and K at FlashAttention tile size
 *      (Q blocks of 128 rows, K blocks of 64 rows, one fp32 scale each);
 *   3. S = Q_i8 K_i8^T with INT32 accumulation, dequantized by q_scale*k_scale;
 *   4. online (tiled) softmax in base 2 (sm_scale*log2(e) is folded into
 *      q_scale);
 *   5. O = P V with P and V kept in FP16 (FP32 accumulation on this GPU).
 *
 * Conventions for every call:
 *   - Tensors are CUDA device pointers to contiguous row-major arrays,
 *     [B, heads, L, d] ("HND"), owned by the caller.  The library never frees
 *     or retains them.  fp16 arguments are IEEE binary16 (`__half`), passed as
 *     `void*`.
 *   - Every pointer must be 16-byte aligned.  Q/K/V/out must not overlap.
 *   - d must be 64 or 128; H % Hkv == 0 (query head h reads kv head
 *     h / (H / Hkv)); Lq, Lk >= 1; B, H, Hkv >= 1; sm_scale > 0 and finite.
 *   - Causal masking is bottom-right aligned: key j is visible to query i iff
 *     j <= i + Lk - Lq.  A query row with no visible key produces zeros.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on that stream.
 *   - Argument errors are detected on the host before anything is launched
 *     and return SAGE_ERR_INVALID_ARG / SAGE_ERR_UNSUPPORTED.  A failed launch
 *     or allocation returns SAGE_ERR_CUDA.  Errors inside a kernel (a bounded
 *     wait that gave up) are recorded in a device status word, read by
 *     sage_check_device_status().
 *   - Every call that smooths and quantizes K (sage_quant_qk*, sage_quant_k,
 *     sage_attn_fwd, its _qblock/_ex/_varlen/_host/_noalloc forms and
 *     sage_attn_decode) accepts Lk <= SAGE_MAX_LK and returns
 *     SAGE_ERR_UNSUPPORTED for a longer K, before any launch.
 *   - Inputs must be finite; NaN/Inf inputs give unspecified outputs.
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAGE_API __attribute__((visibility("default")))
#else
#define SAGE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size */
    SAGE_ERR_UNSUPPORTED = 2,   /* d not in {64,128}, or no sm_100 device */
    SAGE_ERR_CUDA = 3,          /* a CUDA launch, allocation or copy failed */
    SAGE_ERR_TIMEOUT = 4        /* a kernel's bounded wait gave up */
} sage_status;

/* Quantization block sizes (rows per block along the token axis). */
#define SAGE_Q_BLOCK 128
#define SAGE_K_BLOCK 64

/* Longest K (keys per (batch, kv head)) the quantizing calls accept. */
#define SAGE_MAX_LK (1 << 20)

/* Flags of the _ex entry points. */
#define SAGE_PV_ACCUM_F16 1u  /* accumulate P V in fp16 (the article's choice) */
#define SAGE_PV_FP8 2u        /* P and V in FP8 E4M3, fp32 sums (SageAttention2) */

/*
 * sage_quant_qk -- steps 1-2: smoothing of K and per-block INT8 quantization.
 *
 *   q        fp16 [B, H, Lq, d]            (in)
 *   k        fp16 [B, Hkv, Lk, d]          (in)
 *   q_i8     int8 [B, H, Lq, d]            (out)
 *   k_i8     int8 [B, Hkv, Lk, d]          (out) quantized K - mean(K)
 *   q_scale  fp32 [B, H, ceil(Lq/128)]     (out) fl32(fl32(amax/127) * c),
 *                                          c = fl32(double(sm_scale)*log2(e))
 *   k_scale  fp32 [B, Hkv, ceil(Lk/64)]    (out) fl32(amax/127)
 *   k_mean   fp32 [B, Hkv, d]              (out) mean of K over all Lk tokens
 *
 * Needs no scratch memory: the K mean is reduced exactly in on-chip
 * distributed shared memory.  Lk may be at most SAGE_MAX_LK (2^20) keys: a
 * longer K returns SAGE_ERR_UNSUPPORTED before anything is launched (the
 * exact per-thread column sums of the K mean are sized for it).
 * Per block: a = max|x|, r = fl32(127/a), q = clamp(rne(fl32(x*r)), -127, 127);
 * an all-zero block gives q = 0 and scale 0.  For K, x = fl32(float(K) - m),
 * m = fl32(double(sum_t int64(K*2^24)) * 2^-24 / Lk), exact and
 * order-independent, so results are bit-reproducible.
 */
SAGE_API sage_status sage_quant_qk(const void *q, const void *k,
                          int8_t *q_i8, int8_t *k_i8,
                          float *q_scale, float *k_scale, float *k_mean,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          float sm_scale, void *stream);

/*
 * sage_quant_qk_qblock -- sage_quant_qk with a finer Q granularity.
 *
 * The list of techniques in "Berkeley AI 转发研究注意力计算 8 位、4 位量化可对齐
 * FP32 精度基线" (the key-points list) and the SageAttention2 entry of the
 * INT4 search results page name quantization blocks smaller than the
 * attention tile; here Q blocks of q_block_rows rows, one of 128 (the tile,
 * identical to sage_quant_qk), 64, 32 or 1 (one scale per query token).
 * Every block lies inside one 128-row attention tile, so the tiles and the
 * kernels that consume them are unchanged; only the number of Q scales
 * grows.  K keeps its 64-row blocks.
 *
 *   q_scale  fp32 [B, H, ceil(Lq/q_block_rows)]  (out) same formula per block
 *   every other argument: as sage_quant_qk.
 * Returns SAGE_ERR_INVALID_ARG for any other q_block_rows.
 */
SAGE_API sage_status sage_quant_qk_qblock(const void *q, const void *k,
                          int8_t *q_i8, int8_t *k_i8,
                          float *q_scale, float *k_scale, float *k_mean,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          float sm_scale, int q_block_rows, void *stream);

/*
 * sage_quant_k -- steps 1-2 alone: K smoothing (mean over each (batch, kv
 * head)'s Lk tokens, the SageAttention article's K smoothing step, method
 * section) and INT8 quantization of the smoothed K in 64-row blocks, with
 * the same codes, scales and mean as sage_quant_qk produces for K (one
 * launch of K clusters only).  For a K that is quantized once and attended
 * many times, e.g. a key cache for the decoding calls.
 *   k        fp16 [B, Hkv, Lk, d]          (in)
 *   k_i8     int8 [B, Hkv, Lk, d]          (out)
 *   k_scale  fp32 [B, Hkv, ceil(Lk/64)]    (out)
 *   k_mean   fp32 [B, Hkv, d]              (out)
 * No scratch memory.  Errors (and the Lk limit): as sage_quant_qk.
 */
SAGE_API sage_status sage_quant_k(const void *k, int8_t *k_i8, float *k_scale, float *k_mean,
                          int B, int Hkv, int Lk, int d, void *stream);

/*
 * sage_attn_fwd_prequant -- steps 3-5 on already-quantized Q/K: one fused
 * kernel (TMA -> tcgen05 INT8 QK^T into tensor memory -> dequant + exp2
 * online softmax -> FP16 P into tensor memory -> tcgen05 FP16 P.V).
 *
 *   q_i8, k_i8, q_scale, k_scale   as produced by sage_quant_qk
 *   v     fp16 [B, Hkv, Lk, d]     (in)
 *   out   fp16 [B, H, Lq, d]       (out) O = softmax(S) V, rounded to fp16
 *   causal  0 or 1
 * Needs no scratch memory.
 */
SAGE_API sage_status sage_attn_fwd_prequant(const int8_t *q_i8, const int8_t *k_i8,
                                   const float *q_scale, const float *k_scale,
                                   const void *v, void *out,
                                   int B, int H, int Hkv, int Lq, int Lk, int d,
                                   int causal, void *stream);

/*
 * sage_attn_fwd_prequant_qblock -- sage_attn_fwd_prequant for Q quantized by
 * sage_quant_qk_qblock with the same q_block_rows (128, 64, 32 or 1): row i
 * of head (b, h) is dequantized with q_scale[b, h, i / q_block_rows].
 * Returns SAGE_ERR_INVALID_ARG for any other q_block_rows.
 */
SAGE_API sage_status sage_attn_fwd_prequant_qblock(const int8_t *q_i8, const int8_t *k_i8,
                                   const float *q_scale, const float *k_scale,
                                   const void *v, void *out,
                                   int B, int H, int Hkv, int Lq, int Lk, int d,
                                   int causal, int q_block_rows, void *stream);

/*
 * sage_attn_fwd -- the whole forward pass (steps 1-5) on fp16 Q, K, V.
 *   q fp16 [B, H, Lq, d], k/v fp16 [B, Hkv, Lk, d], out fp16 [B, H, Lq, d].
 * Scratch (int8 Q/K, scales, mean, partial sums;
 * sage_workspace_size() bytes) is allocated with cudaMallocAsync on
 * `stream` and released with cudaFreeAsync on the same stream.
 */
SAGE_API sage_status sage_attn_fwd(const void *q, const void *k, const void *v, void *out,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          int causal, float sm_scale, void *stream);

/*
 * sage_attn_fwd_qblock -- sage_attn_fwd with Q quantized in blocks of
 * q_block_rows rows (128, 64, 32 or 1; see sage_quant_qk_qblock).  Its
 * scratch, allocated and released on `stream` like sage_attn_fwd's, is at
 * most sage_workspace_size() + 4*B*H*Lq + 256 bytes (the Q scales grow
 * to ceil(Lq/q_block_rows) per head).
 */
SAGE_API sage_status sage_attn_fwd_qblock(const void *q, const void *k, const void *v, void *out,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          int causal, float sm_scale, int q_block_rows, void *stream);

/*
 * sage_attn_fwd_ex / sage_attn_fwd_prequant_ex -- the _qblock entry points
 * with a flags word.  SAGE_PV_ACCUM_F16 selects the P V accumulator the
 * SageAttention article states (an fp16 accumulator, method section, FP16
 * P V step): P and V stay fp16 and their products are summed in fp16
 * (the tensor core's F16 D format) instead of fp32.  With it the running
 * row max is kept exact (O is rescaled whenever it grows), so P <= 1 and, as
 * the article argues, the sums stay within the fp16 range; the result is
 * less accurate than the fp32 default (the error grows with Lk) and no
 * faster on this GPU.  SAGE_PV_FP8 (sage_attn_fwd_ex only) quantizes V to
 * E4M3 per channel (sage_quant_v_fp8) and P to E4M3 and runs P V on the FP8
 * tensor-core path with fp32 sums, as the SageAttention2 description (INT4
 * search results page, SageAttention2 entry) proposes.  flags = 0 is
 * identical to the _qblock calls.  Any other value, both bits together, or
 * SAGE_PV_FP8 given
 * to sage_attn_fwd_prequant_ex (which takes fp16 V; use
 * sage_attn_fwd_prequant_fp8pv) returns SAGE_ERR_INVALID_ARG.
 */
SAGE_API sage_status sage_attn_fwd_ex(const void *q, const void *k, const void *v, void *out,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          int causal, float sm_scale, int q_block_rows, unsigned flags,
                          void *stream);
SAGE_API sage_status sage_attn_fwd_prequant_ex(const int8_t *q_i8, const int8_t *k_i8,
                                   const float *q_scale, const float *k_scale,
                                   const void *v, void *out,
                                   int B, int H, int Hkv, int Lq, int Lk, int d,
                                   int causal, int q_block_rows, unsigned flags, void *stream);

/*
 * sage_quant_qk_varlen / sage_attn_fwd_prequant_varlen / sage_attn_fwd_varlen
 * -- the _qblock / _ex calls on a padded batch whose entries hold different
 * numbers of query rows and keys.  Entry b uses rows [0, seqlens_q[b]) of its
 * [Lq, d] Q rows and keys [0, seqlens_k[b]) of its [Lk, d] K/V rows
 * (seqlens_q, seqlens_k: device int32 [B], values clamped to [0, Lq] and
 * [0, Lk]; either pointer may be NULL, meaning every entry uses all Lq rows or
 * all Lk keys).  Each entry is then computed exactly as the same call on that
 * entry alone with Lq = seqlens_q[b], Lk = seqlens_k[b]: K smoothing
 * (step 1 of the SageAttention article's method) subtracts the mean over the
 * entry's own keys, the last Q and K blocks of an entry are ragged, causal
 * masking is bottom-right aligned to (seqlens_q[b], seqlens_k[b]).
 *
 * Padding is not read and not written by the quantization (its int8 rows and
 * scales keep whatever the buffers held).  The attention kernels write zeros
 * to the output rows past seqlens_q[b] and never give weight to a key past
 * seqlens_k[b].  On the fp16 P V paths, V rows in
 * [seqlens_k[b], 64 * ceil(seqlens_k[b] / 64)), the rest of an entry's last
 * 64-key tile, are multiplied by zero weights and must therefore hold finite
 * values (zeros, say): an Inf or NaN there turns the entry's output into
 * NaN.  An entry with no rows or no keys outputs zeros.
 *
 * flags: as sage_attn_fwd_ex / sage_attn_fwd_prequant_ex.  With SAGE_PV_FP8
 * (sage_attn_fwd_varlen only) each entry's per-channel V scales span its own
 * keys and the E4M3 codes past seqlens_k[b] are 0, so on that path V's
 * padding is never read and need not be finite.
 * Every other argument, layout, error and scratch rule: as the call named.
 */
SAGE_API sage_status sage_quant_qk_varlen(const void *q, const void *k,
                          int8_t *q_i8, int8_t *k_i8,
                          float *q_scale, float *k_scale, float *k_mean,
                          const int *seqlens_q, const int *seqlens_k,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          float sm_scale, int q_block_rows, void *stream);
SAGE_API sage_status sage_attn_fwd_prequant_varlen(const int8_t *q_i8, const int8_t *k_i8,
                                   const float *q_scale, const float *k_scale,
                                   const void *v, void *out,
                                   const int *seqlens_q, const int *seqlens_k,
                                   int B, int H, int Hkv, int Lq, int Lk, int d,
                                   int causal, int q_block_rows, unsigned flags, void *stream);
SAGE_API sage_status sage_attn_fwd_varlen(const void *q, const void *k, const void *v,
                          void *out, const int *seqlens_q, const int *seqlens_k,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          int causal, float sm_scale, int q_block_rows, unsigned flags,
                          void *stream);

/*
 * sage_quant_v_fp8 -- V to FP8 E4M3 with one scale per channel over all Lk
 * tokens of a (batch, kv head): a = max_t |V[t, c]|, r = fl32(448 / a),
 * code = e4m3(fl32(V * r)) (round to nearest even, saturating at 448),
 * scale = fl32(a / 448); a zero channel gives codes 0 and scale 0.
 *   v        fp16 [B, Hkv, Lk, d]                      (in)
 *   v8t      uint8 [B, Hkv, d, Lkp], Lkp = 64*ceil(Lk/64) (out) E4M3 codes,
 *            channel-major (keys contiguous); positions >= Lk hold 0
 *   v_scale  fp32 [B, Hkv, d]                          (out)
 *   workspace: sage_quant_v_fp8_workspace_size() bytes or NULL/0 (allocated
 *   with cudaMallocAsync on `stream`).
 */
SAGE_API sage_status sage_quant_v_fp8(const void *v, uint8_t *v8t, float *v_scale,
                                      int B, int Hkv, int Lk, int d,
                                      void *workspace, size_t workspace_bytes, void *stream);
SAGE_API size_t sage_quant_v_fp8_workspace_size(int B, int Hkv, int d);

/*
 * sage_attn_fwd_prequant_fp8pv -- steps 3-5 with P and V in FP8 E4M3: V from
 * sage_quant_v_fp8 (v8t, v_scale), P = e4m3(1.75 * p) with p relative to the
 * running row max (p <= 2^8), P V on the tensor core's FP8 path with fp32
 * sums, the row sum taken over the unquantized p.  Other arguments as
 * sage_attn_fwd_prequant_qblock.
 */
SAGE_API sage_status sage_attn_fwd_prequant_fp8pv(const int8_t *q_i8, const int8_t *k_i8,
                                   const float *q_scale, const float *k_scale,
                                   const uint8_t *v8t, const float *v_scale, void *out,
                                   int B, int H, int Hkv, int Lq, int Lk, int d,
                                   int causal, int q_block_rows, void *stream);

/*
 * sage_attn_decode_prequant -- steps 3-5 for a few query tokens against a
 * long key sequence (decoding against a KV cache): the same arithmetic as
 * sage_attn_fwd_prequant, laid out for Lq << Lk.  The H / Hkv query heads of
 * a kv head are packed into one 128-row tile, so each K/V tile is read from
 * HBM once per kv head, and the keys are split over several CTAs whose
 * partial results a second kernel merges (the merge is skipped when one
 * split suffices).  Requires (H / Hkv) * Lq <= 128, else returns
 * SAGE_ERR_UNSUPPORTED (use sage_attn_fwd_prequant_qblock).
 *   q_i8, k_i8, q_scale, k_scale   as produced by sage_quant_qk_qblock with
 *                                  the same q_block_rows
 *   v, out, causal                 as sage_attn_fwd_prequant (bottom-right
 *                                  causal alignment)
 *   workspace, workspace_bytes     device scratch of at least
 *                                  sage_attn_decode_workspace_size() bytes for
 *                                  the partial results, or NULL/0 to let the
 *                                  call allocate it with cudaMallocAsync on
 *                                  `stream`.
 * The article has no separate decoding kernel; this is the forward pass of
 * its method for the GQA / long-context serving case it names.
 */
SAGE_API sage_status sage_attn_decode_prequant(const int8_t *q_i8, const int8_t *k_i8,
                                   const float *q_scale, const float *k_scale,
                                   const void *v, void *out,
                                   int B, int H, int Hkv, int Lq, int Lk, int d,
                                   int causal, int q_block_rows,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * sage_attn_decode_prequant_varlen -- sage_attn_decode_prequant for a batch
 * whose entries hold different numbers of keys in one padded cache: entry b
 * uses keys [0, seqlens_k[b]) of its [Lk, d] rows (seqlens_k: device int32
 * [B], values clamped to [0, Lk]; key blocks and their k_scale entries past an
 * entry's length are not read).  Causal masking is bottom-right aligned to
 * seqlens_k[b]; an entry with no keys outputs zeros.  K of each entry must
 * have been smoothed and quantized over its own keys (its own mean).
 */
SAGE_API sage_status sage_attn_decode_prequant_varlen(const int8_t *q_i8, const int8_t *k_i8,
                                   const float *q_scale, const float *k_scale,
                                   const void *v, void *out, const int *seqlens_k,
                                   int B, int H, int Hkv, int Lq, int Lk, int d,
                                   int causal, int q_block_rows,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * sage_attn_decode_prequant_paged -- the decoding layout on a paged cache.
 * A page holds 64 consecutive keys (one K quantization block) of every kv
 * head: k_pages int8 [num_pages, Hkv, 64, d], v_pages fp16 [num_pages, Hkv,
 * 64, d], k_scale_pages fp32 [num_pages, Hkv] (the scale of that block).
 * block_table int32 [B, max_blocks] (device) lists entry b's pages in key
 * order; seqlens_k int32 [B] (device) its key counts (clamped to
 * [0, 64 * max_blocks]); page indices outside [0, num_pages) are clamped.
 * q_i8, q_scale, out, causal, q_block_rows, workspace: as
 * sage_attn_decode_prequant with Lk = 64 * max_blocks (also for
 * sage_attn_decode_workspace_size).  K of each entry must have been smoothed
 * and quantized over its own keys.
 */
SAGE_API sage_status sage_attn_decode_prequant_paged(const int8_t *q_i8, const float *q_scale,
                                   const int8_t *k_pages, const float *k_scale_pages,
                                   const void *v_pages, const int *block_table,
                                   const int *seqlens_k, void *out,
                                   int B, int H, int Hkv, int Lq, int num_pages, int max_blocks,
                                   int d, int causal, int q_block_rows,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of scratch sage_attn_decode_prequant needs (0 for unsupported shapes). */
SAGE_API size_t sage_attn_decode_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int d);

/*
 * sage_attn_decode -- quantization (sage_quant_qk_qblock) followed by
 * sage_attn_decode_prequant on fp16 q, k, v; scratch allocated with
 * cudaMallocAsync on `stream` and released on the same stream.
 */
SAGE_API sage_status sage_attn_decode(const void *q, const void *k, const void *v, void *out,
                          int B, int H, int Hkv, int Lq, int Lk, int d,
                          int causal, float sm_scale, int q_block_rows, void *stream);

/*
 * sage_attn_fwd_host -- sage_attn_fwd on HOST buffers, for callers whose data
 * lives in host memory.  q/k/v/out are host pointers with the layouts of
 * sage_attn_fwd (pinned memory gives asynchronous copies; pageable memory
 * works but the copies then block the calling thread).  On `stream` the call
 * allocates device buffers (cudaMallocAsync) and frees them after the work;
 * in between the (batch, kv head) groups are processed in up to 8 chunks
 * through a three-stage pipeline on internal streams (copy in, compute, copy
 * out; ordered after `stream`, and `stream` after them), so the copies of
 * later chunks overlap the kernels of earlier ones.  The output is that of
 * sage_attn_fwd, bit for bit.  The host output is valid once `stream` has been
 * synchronized; the host buffers must stay alive until then.
 */
SAGE_API sage_status sage_attn_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                               void *out_host, int B, int H, int Hkv, int Lq, int Lk, int d,
                               int causal, float sm_scale, void *stream);

/*
 * sage_attn_fwd_host_qblock -- sage_attn_fwd_host with Q quantized in blocks
 * of q_block_rows rows (128, 64, 32 or 1; see sage_quant_qk_qblock); the
 * output is that of sage_attn_fwd_qblock, bit for bit.  Any other
 * q_block_rows returns SAGE_ERR_INVALID_ARG.
 */
SAGE_API sage_status sage_attn_fwd_host_qblock(const void *q_host, const void *k_host,
                               const void *v_host, void *out_host,
                               int B, int H, int Hkv, int Lq, int Lk, int d,
                               int causal, float sm_scale, int q_block_rows, void *stream);

/*
 * sage_attn_fwd_noalloc -- sage_attn_fwd for callers that must not allocate
 * device memory at call time (a serving process that reserved its whole
 * memory budget at start-up and treats any later allocation as an error, or a
 * plugin host that gives the library no allocator).  The article has no
 * counterpart; this is a packaging variant of the same forward pass.
 *   Arguments, layouts and results are those of sage_attn_fwd.  The scratch
 *   lives in one fixed 64 MiB device array inside the library, reserved on
 *   every GPU that loads that part of the library and held until exit.
 *   Problems needing more scratch than that (sage_workspace_size() >
 *   64 MiB) return SAGE_ERR_INVALID_ARG without launching anything.
 *   All calls share the array: calls whose kernels overlap on the GPU race
 *   and give wrong results, so order them on one stream.  The first call on
 *   each device (and the first after its context was destroyed and created
 *   again, e.g. by cudaDeviceReset) looks the array up; make it before any
 *   stream capture begins.  Nothing in the array needs clearing between
 *   calls.  Shapes, pointers, scalars and the Lk limit are checked as for
 *   sage_attn_fwd, and sage_last_launch_count() reports the kernels a
 *   successful call launched.
 */
SAGE_API sage_status sage_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                           void *out, int B, int H, int Hkv, int Lq, int Lk,
                                           int d, int causal, float sm_scale, void *stream);

/*
 * sage_workspace_size -- bytes of device scratch sage_attn_fwd allocates for
 * one call on this shape (int8 Q and K, their block scales and the K mean,
 * each piece 256-byte aligned); 0 for a shape the calls reject.
 */
SAGE_API size_t sage_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int d);

/*
 * sage_check_device_status -- synchronizes `stream`, then reports and clears
 * the device status word: SAGE_ERR_TIMEOUT if any kernel launched since the
 * last check gave up on a bounded wait (its outputs are then invalid),
 * SAGE_ERR_CUDA if the synchronization itself failed, else SAGE_OK.
 */
SAGE_API sage_status sage_check_device_status(void *stream);

/*
 * sage_debug_wait_timeout -- diagnostic with no counterpart in the article:
 * launches on `stream` a one-warp kernel that waits, through the same bounded
 * wait the attention kernel uses, on a barrier that nothing ever completes.
 * After limit_ms (1..2000) the wait gives up and records the event, so the
 * next sage_check_device_status(stream) returns SAGE_ERR_TIMEOUT (and clears
 * it).  Used to test the error path without faulting or hanging the GPU.
 * Returns SAGE_ERR_INVALID_ARG for limit_ms outside 1..2000.
 */
SAGE_API sage_status sage_debug_wait_timeout(int limit_ms, void *stream);

/* Static, human-readable name of a status code. */
SAGE_API const char *sage_status_string(sage_status s);

/* Number of kernels the last successful call on this thread launched. */
SAGE_API int sage_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_B200_H */
