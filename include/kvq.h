/*
 * kvq.h -- C ABI of libkvq: KV-cache compression and one decode step over the
 * compressed cache, hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 *  - All data pointers are DEVICE pointers owned by the caller.  The library never
 *    allocates or frees memory and never synchronises the stream; it keeps no state
 *    between calls other than cached device properties.
 *  - Calls are asynchronous: KVQ_OK means the work was enqueued on `stream`
 *    (NULL = the legacy default stream) of the current device.  A fault inside a
 *    kernel surfaces on the caller's next synchronisation.
 *  - Arguments are validated on the host before anything is launched; a failed check
 *    returns its error code and enqueues nothing.  Zero rows/keys return KVQ_OK with
 *    no launch.
 *  - KVQ_ERR_CUDA means the CUDA runtime reported an error when the kernel was
 *    launched (this can also be a sticky error left by earlier asynchronous work).
 *  - fp16 data is passed as raw IEEE binary16 bit patterns (uint16_t).
 *  - Rows are contiguous and row-major; 64-bit sizes are used throughout.
 *  - No C++ exception crosses this boundary.
 *
 * Sources (web pages, cited by title and section):
 *  [INT8]  "Q-TensorFormer" model card, section 6 "Adaptive KV Cache Quantization &
 *          Attention-Sink Eviction": symmetric INT8, X_hat = clamp(round(X/s8), -128,
 *          127) * s8 with s8 = max|X| / 127.
 *  [PAPER] "GPU-Accelerated INT8 Quantization for KV Cache Compression in Large
 *          Language Models" (arXiv 2601.04719), abstract.
 *  [QJL]   "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with Zero
 *          Overhead" (arXiv 2406.03482), abstract.
 *  [GQA]   "Q-TensorFormer" model card, section 4 "Grouped-Query Attention (GQA) &
 *          Multi-Query Attention (MQA)".
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, spelled without CUDA headers. */
typedef struct CUstream_st* kvq_stream_t;

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size, bad enum ... */
    KVQ_ERR_UNSUPPORTED = 2,   /* a valid request this build does not implement       */
    KVQ_ERR_CUDA = 3,          /* the CUDA runtime reported an error at launch         */
    KVQ_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required           */
    KVQ_ERR_DEVICE = 5         /* a kernel recorded a device-side error (see below)    */
} kvq_status;

typedef enum { KVQ_F32 = 0, KVQ_F16 = 1 } kvq_dtype;

typedef enum { KVQ_KEYS_INT8 = 0, KVQ_KEYS_QJL = 1 } kvq_key_format;

#define KVQ_ABI_VERSION 2

int kvq_abi_version(void);
const char* kvq_status_string(kvq_status s);

/*
 * kvq_quantize_int8 -- [INT8] with one scale per row ("per token": a row is one head's
 * head_dim vector); [PAPER] abstract (INT8 KV quantization, 4x smaller than fp32).
 *   For each row r:  a_r = max_j |x_rj|,   s_r = fl32(a_r / 127),
 *                    c_rj = clamp(round_half_even(fl32(x_rj / s_r)), -128, 127),
 *   where the quotient is an IEEE fp32 division by the STORED scale; a row with
 *   s_r == 0 gets codes 0.  (|x/s| <= 127 whenever s is a normal number, so the clamp
 *   only binds for rows whose scale is subnormal.)  Results are bit-exact.
 *   x       [n_rows][d] fp32 or fp16 (x_dtype), 16-byte aligned
 *   codes   [n_rows][d] int8, 16-byte aligned         (written)
 *   scales  [n_rows]    fp32, 4-byte aligned          (written)
 *   d       > 0, multiple of 16, <= 65536
 *   NaN/Inf inputs give unspecified codes (not checked).
 */
kvq_status kvq_quantize_int8(const void* x, kvq_dtype x_dtype, int64_t n_rows, int64_t d,
                             int8_t* codes, float* scales, kvq_stream_t stream);

/*
 * kvq_dequantize_int8 -- [INT8] the trailing "* s8": x_hat_rj = fl32(c_rj * s_r); for
 * fp16 output, that fp32 value rounded to nearest-even fp16.  Bit-exact.
 *   codes [n_rows][d] int8 (16-byte aligned), scales [n_rows] fp32,
 *   out   [n_rows][d] fp32 or fp16 (out_dtype), 16-byte aligned (written);
 *   d > 0, multiple of 16.
 */
kvq_status kvq_dequantize_int8(const int8_t* codes, const float* scales, int64_t n_rows,
                               int64_t d, void* out, kvq_dtype out_dtype, kvq_stream_t stream);

/*
 * kvq_int8_scores -- [PAPER] "attention score" of one query against INT8 rows:
 *   scores_r = sum_j q_j * fl32(c_rj * s_r), fp32 accumulation (order unspecified).
 *   q [d] fp32 or fp16 (q_dtype, 16-byte aligned), codes [n_rows][d] int8 (16-byte
 *   aligned), scales [n_rows] fp32, scores [n_rows] fp32 (written); d multiple of 16,
 *   d <= 16384.
 */
kvq_status kvq_int8_scores(const void* q, kvq_dtype q_dtype, const int8_t* codes,
                           const float* scales, int64_t n_rows, int64_t d, float* scores,
                           kvq_stream_t stream);

/*
 * kvq_qjl_encode -- [QJL] abstract ("a JL transform followed by sign-bit quantization"):
 *   u_n = S k_n for each key (fp16 x fp16 products, fp32 accumulation on the tensor
 *   cores); bit i of key n = [u_n,i >= 0], stored LSB-first, 32 coordinates per word
 *   (word w holds coordinates 32w .. 32w+31); norm_n = fp16(||k_n||_2).
 *   keys_f16    [n_keys][d] fp16, 16-byte aligned
 *   sketch_f16  [m][d] fp16 row-major (the Gaussian JL matrix S), 16-byte aligned
 *   sign_words  [n_keys][m/32] uint32 (written), 16-byte aligned if m/32 is a multiple
 *               of 4, else 4-byte aligned
 *   norms_f16   [n_keys] fp16 (written), 2-byte aligned
 *   d must be 128 and m a multiple of 32 in [32, 256] (else KVQ_ERR_UNSUPPORTED).
 *   A bit may differ from the exact (fp64) sign only where |u_i| is within the fp32
 *   accumulation error of 0.
 */
kvq_status kvq_qjl_encode(const uint16_t* keys_f16, int64_t n_keys, int32_t d,
                          const uint16_t* sketch_f16, int32_t m, uint32_t* sign_words,
                          uint16_t* norms_f16, kvq_stream_t stream);

/*
 * kvq_qjl_query_sketch -- [QJL] abstract ("a standard JL transform without
 * quantization to the other [vector]"): v_n = S q_n in fp32 (tensor cores).
 *   q_f16 [n_q][d] fp16 (16-byte aligned), sketch_f16 [m][d] fp16 (16-byte aligned),
 *   v [n_q][m] fp32 (written, 16-byte aligned); d == 128, m multiple of 32 in [32, 256].
 */
kvq_status kvq_qjl_query_sketch(const uint16_t* q_f16, int64_t n_q, int32_t d,
                                const uint16_t* sketch_f16, int32_t m, float* v,
                                kvq_stream_t stream);

/*
 * kvq_decode_attention -- one decode step for one query token per head over a
 * compressed cache ([PAPER] abstract: attention scores over the INT8 cache; [QJL]
 * abstract: the asymmetric estimator; [GQA] section 4: query head h reads KV head
 * h / (Hq / Hkv)).
 *   score_t = INT8 keys: sum_j q_j * fl32(c_tj * s_t);
 *             QJL keys:  sqrt(pi/2)/m * norm_t * sum_i v_i * (2 b_t,i - 1), v = S q (fp32);
 *   p_t     = softmax_t(sm_scale * score_t) over all T cached tokens (no mask);
 *   out     = sum_t p_t * fl32(cv_t * sv_t)   (fp32, [B][Hq][D]).
 * Layouts (all contiguous):
 *   q          [B][Hq][D] fp16
 *   k_codes    [B][Hkv][T][D] int8,  k_scales [B][Hkv][T] fp32      (INT8 keys)
 *   k_words    [B][Hkv][T][m/32] u32, k_norms [B][Hkv][T] fp16,
 *   sketch     [m][D] fp16                                          (QJL keys)
 *   v_codes    [B][Hkv][T][D] int8,  v_scales [B][Hkv][T] fp32      (needed if out)
 *   out        [B][Hq][D] fp32 or NULL
 *   scores_out [B][Hq][T] fp32 raw scores (before sm_scale) or NULL
 * out and scores_out may not both be NULL.  head_dim must be 128 (KVQ_ERR_UNSUPPORTED
 * otherwise); QJL needs m a multiple of 32 in [32, 256]; Hq % Hkv == 0, any group size
 * G = Hq / Hkv (MHA G = 1, GQA, MQA Hkv = 1); T >= 1 (a softmax over no tokens is
 * undefined: KVQ_ERR_INVALID_ARG).  sm_scale == 0 selects 1/sqrt(head_dim).
 * Group sizes: one CTA serves up to 8 query heads of a KV head with INT8 keys and up
 * to 4 with QJL keys (the largest power of two dividing G); a larger G is served by
 * G / that CTAs per token range, which stream the same cache bytes side by side (the
 * second read mostly from L2).
 * Precision: scores and the softmax in fp32 (exponentials by the hardware 2^x); out
 * within 2e-3 absolute of the fp64 value of the formula above.  Unless
 * KVQ_DECODE_CUDA_CORES is set, the contractions run on the tensor cores where they
 * apply, as exact integer products:
 *   QJL keys (T a multiple of 8, k_words and v_codes 16-byte aligned, at most 9 units
 *   per CTA range, fewer than 2^31 token rows): the weighted sum, per chunk of 128 tokens
 *   and head, with the weights p_t * sv_t relative to the chunk's largest p as integers
 *   in units of 2^-E, smax 2^E in [2^23, 2^24) for the chunk's largest value scale smax,
 *   multiplying the INT8 codes exactly in int32 (error below 2^-23 smax per token: the
 *   product p_t * sv_t is rounded to fp32 before its rounding to the fixed point);
 *   INT8 keys (T >= 512, k_codes and v_codes 16-byte aligned, at most 4 units per CTA
 *   range, fewer than 2^31 token rows): the scores, as exact int32 sums of the key codes
 *   times the query written as the fixed-point integer round(q 2^E), max|q| 2^E in
 *   [2^21, 2^22) (error at most 2^-22 max|q| per query entry), rounded once to fp32 and
 *   multiplied by s_t; and the weighted sum as for QJL keys, per block of 32 tokens.
 * Everything else runs in fp32 on the CUDA cores.
 * flags (KVQ_DECODE_*): KVQ_DECODE_CUDA_CORES keeps the whole step on the CUDA cores
 * (fp32 scores and weighted sum even where the tensor-core kernels apply); 0 lets the
 * library choose; KVQ_DECODE_TEST_EXPIRE is for testing the failure path (below the
 * struct); other bits: KVQ_ERR_INVALID_ARG.
 * workspace: caller-owned device memory of at least kvq_decode_workspace_bytes(a)
 * bytes, 256-byte aligned (KVQ_ERR_WORKSPACE otherwise).  It holds per-split partial
 * softmax states and, for QJL keys, the query projections; its contents on entry do not
 * matter.
 * Launches 2 kernels (the decode and the merge of its partial states), 3 with QJL keys
 * on the CUDA cores (the query projections first), on `stream`; no host synchronisation.
 * If a decode kernel records a device-side error (see kvq_device_error), the outputs of
 * this and of every later decode call are NaN until kvq_device_error() reads and clears
 * the error: out is valid only while kvq_device_error() reports 0.
 */
typedef struct kvq_decode_args {
    int64_t batch;
    int64_t n_q_heads;
    int64_t n_kv_heads;
    int64_t seq_len;
    int32_t head_dim;
    int32_t key_format;            /* kvq_key_format */
    const uint16_t* q_f16;
    const int8_t* k_codes;
    const float* k_scales;
    const uint32_t* k_words;
    const uint16_t* k_norms_f16;
    const uint16_t* sketch_f16;
    int32_t sketch_dim;            /* m */
    float sm_scale;
    const int8_t* v_codes;
    const float* v_scales;
    float* out;
    float* scores_out;
    void* workspace;
    size_t workspace_bytes;
    uint32_t flags;                /* KVQ_DECODE_* */
} kvq_decode_args;

#define KVQ_DECODE_CUDA_CORES 1u   /* no tensor-core contraction */
/* For testing the failure path only: the tensor-core decode kernels issue none of their
 * key loads, so the bounded waits of the roles that consume them expire (after about 2 s
 * each): the call completes, kvq_device_error() then reports the kernel's code, and the
 * outputs are NaN.  No fault and no hang: every wait is bounded.  The CUDA-core kernels
 * ignore it. */
#define KVQ_DECODE_TEST_EXPIRE 2u

kvq_status kvq_decode_attention(const kvq_decode_args* a, kvq_stream_t stream);

/* Bytes of workspace kvq_decode_attention needs for these arguments (0 if the
 * arguments are invalid).  Depends on the current device's SM count. */
size_t kvq_decode_workspace_bytes(const kvq_decode_args* a);

/*
 * kvq_quantize_int8_channelwise / kvq_dequantize_int8_channelwise -- the symmetric INT8
 * equation of kvq_quantize_int8 with one scale per channel ("Q-TensorFormer" model
 * card, section 6, Symmetric Channel-Wise INT8: X_hat = clamp(round(X / s8), -128, 127)
 * * s8, s8 = max|X| / 127).  x holds n_blocks blocks of [rows][d] row-major, one block
 * after another (for a KV cache [B][H][T][D]: n_blocks = B * H, rows = T); for block b
 * and column j:
 *   s[b][j] = fl32(max_r |x[b][r][j]| / 127),
 *   codes[b][r][j] = clamp(rint_even(fl32(x[b][r][j] / s[b][j])), -128, 127)  (0 if s = 0);
 *   dequantize: out = fl32(codes * s) (fp16 out: that value rounded to nearest even).
 * Bit-identical to that definition.  d must be a multiple of 64, rows >= 1; x, codes,
 * out 16-byte aligned, scales [n_blocks][d] 4-byte aligned (else KVQ_ERR_INVALID_ARG);
 * n_blocks <= 65535 and rows * d < 2^35 (else KVQ_ERR_UNSUPPORTED).
 * n_blocks == 0: no launch.  One launch each; stream-ordered, no synchronisation.
 */
kvq_status kvq_quantize_int8_channelwise(const void* x, kvq_dtype x_dtype, int64_t n_blocks, int64_t rows,
                                         int64_t d, int8_t* codes, float* scales, kvq_stream_t stream);
kvq_status kvq_dequantize_int8_channelwise(const int8_t* codes, const float* scales, int64_t n_blocks,
                                           int64_t rows, int64_t d, void* out, kvq_dtype out_dtype,
                                           kvq_stream_t stream);

/*
 * kvq_quantize_int4 / kvq_dequantize_int4 -- asymmetric group-wise INT4 ("Q-TensorFormer"
 * model card, section 6, Asymmetric Group-Wise INT4: X_hat = clamp(round((X - z4) / s4),
 * 0, 15) * s4 + z4, s4 = (max X - min X) / 15, z4 = min X).  x: [n_rows][d] fp32 or fp16;
 * each row is cut into groups of `group` consecutive elements (32, 64 or 128; d a
 * multiple of it).  Per group g of row r, in fp32 with IEEE operations:
 *   z = min x,  s = fl32(fl32(max x - min x) / 15),
 *   c = clamp(rint_even(fl32(fl32(x - z) / s)), 0, 15)  (0 if s = 0),
 *   dequantize: out = fl32(fl32(c * s) + z) (fp16 out: rounded to nearest even).
 * packed: [n_rows][d/2] bytes, element 2i in bits 0-3 and 2i+1 in bits 4-7;
 * scales, zeros: [n_rows][d/group] fp32.  Bit-identical to the definition.  x and out
 * 16-byte aligned, packed 16-byte aligned (quantize) or 4-byte aligned (dequantize),
 * scales/zeros 4-byte aligned (else KVQ_ERR_INVALID_ARG); other group sizes
 * KVQ_ERR_UNSUPPORTED.  One launch each.
 */
kvq_status kvq_quantize_int4(const void* x, kvq_dtype x_dtype, int64_t n_rows, int64_t d, int32_t group,
                             uint8_t* packed, float* scales, float* zeros, kvq_stream_t stream);
kvq_status kvq_dequantize_int4(const uint8_t* packed, const float* scales, const float* zeros,
                               int64_t n_rows, int64_t d, int32_t group, void* out, kvq_dtype out_dtype,
                               kvq_stream_t stream);

/*
 * kvq_qjl_residual_encode -- keys as group-wise INT4 plus a 1-bit QJL sketch of the INT4
 * residual: a first quantizer takes most of the bits and a 1-bit Johnson-Lindenstrauss
 * layer corrects its error (the "TurboQuant" news page, "Кризис отменяется: Google
 * изобрел квантовый алгоритм сокращения объема памяти для ИИ в 6 раз", on its two
 * stages; the 1-bit stage is the QJL sketch of kvq_qjl_encode, the first stage the
 * asymmetric group-wise INT4 of kvq_quantize_int4).  Per key k (fp16, d = 128):
 *   packed, scales, zeros = kvq_quantize_int4 of k (groups of `group`), bit-identical;
 *   residual_f16 = fp16(fl32(k - k_hat)), k_hat = fl32(fl32(c * s) + z) (the INT4
 *                  reconstruction), RN; an output, and the input of the sketch stage;
 *   sign_words, rnorms_f16 = kvq_qjl_encode of the residual rows (bits of S r, fp16 of
 *                  ||r||), with the same exactness as kvq_qjl_encode.
 * Scores against such a key (see kvq_decode_attention_qjlres): <q, k_hat> +
 * sqrt(pi/2)/m * ||r|| * sum_i (S q)_i (2 b_i - 1).
 * keys, packed, residual_f16 16-byte aligned, scales/zeros 4-byte, sign_words as in
 * kvq_qjl_encode, rnorms 2-byte (else KVQ_ERR_INVALID_ARG); d and m as kvq_qjl_encode,
 * group 32/64/128 (else KVQ_ERR_UNSUPPORTED).  Two launches (INT4 + residual, then the
 * tensor-core sketch); stream-ordered.
 */
kvq_status kvq_qjl_residual_encode(const uint16_t* keys_f16, int64_t n_keys, int32_t d, int32_t group,
                                   const uint16_t* sketch_f16, int32_t m, uint8_t* packed, float* scales,
                                   float* zeros, uint16_t* residual_f16, uint32_t* sign_words,
                                   uint16_t* rnorms_f16, kvq_stream_t stream);

/*
 * kvq_decode_append -- one decode step that first appends the newly generated token to
 * the compressed cache ("Quantum-Inspired GPU & J-Space VRAM Optimizer" page, section 4,
 * "Framework Integration": the cache writes are intercepted and the compressed
 * representation is stored; the INT8 and QJL encodings are those of
 * kvq_quantize_int8 and kvq_qjl_encode).  For every (batch b, KV head g):
 *   keys   INT8: k_codes/k_scales row T = the per-row absmax INT8 quantization of
 *               k_new[b][g] (bit-identical to kvq_quantize_int8 of that row);
 *          QJL:  k_words row T = sign bits of S k_new[b][g] and k_norms row T =
 *               fp16(||k_new[b][g]||) (as kvq_qjl_encode: the norm bit-identical, the
 *               bits computed in fp32, so a bit may differ from an exact computation
 *               only where |(S k)_i| < 1e-4 ||k||);
 *   values v_codes/v_scales row T = the INT8 quantization of v_new[b][g];
 * then the decode step of kvq_decode_attention over the T + 1 tokens 0 .. T, with the
 * result that step would give on the updated cache.
 *   base:      the decode arguments, with base.seq_len = T >= 0, the tokens already
 *              cached, and the cache arrays laid out [B][Hkv][capacity][...] (unit
 *              stride `capacity` rows instead of seq_len); base.out [B][Hq][D] and/or
 *              base.scores_out [B][Hq][T + 1].  base.out needs base.v_codes/v_scales.
 *   capacity:  rows per (b, KV head) in the cache arrays, >= T + 1; rows other than
 *              0 .. T are neither read nor written.
 *   k_new_f16, v_new_f16: [B][Hkv][D] fp16, 16-byte aligned; v_new_f16 may be NULL
 *              when base.out is NULL (the value rows are then not appended).
 * The appended rows are written before the attention reads them: by a small kernel
 * ahead of the decode where a tensor-core decode kernel runs (see kvq_decode_attention),
 * else by the CUDA-core decode kernel itself in the same launch.  Workspace as
 * kvq_decode_attention, sized by kvq_decode_append_workspace_bytes.  Errors as
 * kvq_decode_attention.
 */
typedef struct kvq_decode_append_args {
    kvq_decode_args base;
    int64_t capacity;
    const uint16_t* k_new_f16;
    const uint16_t* v_new_f16;
} kvq_decode_append_args;

kvq_status kvq_decode_append(const kvq_decode_append_args* a, kvq_stream_t stream);
size_t kvq_decode_append_workspace_bytes(const kvq_decode_append_args* a);

/*
 * kvq_decode_attention_int4v -- the decode step of kvq_decode_attention with INT8 keys
 * and group-wise INT4 values (the layout kvq_quantize_int4 writes; "Q-TensorFormer" model
 * card, section 6): the value row of token t is x_hat = fl32(fl32(c * s4) + z4) per group,
 * out = sum_t p_t x_hat_t.  base as for kvq_decode_attention with INT8 keys, except that
 * base.v_codes / base.v_scales are ignored:
 *   v_packed  [B][Hkv][T][D/2] bytes (element 2i in bits 0-3), 16-byte aligned;
 *   v_scales4, v_zeros4  [B][Hkv][T][D/v_group] fp32, 4-byte aligned;
 *   v_group   32, 64 or 128 (KVQ_ERR_UNSUPPORTED otherwise, and for QJL keys).
 * Workspace from kvq_decode_int4v_workspace_bytes; results and errors as
 * kvq_decode_attention (outputs within fp32 reassociation of the definition: the kernel
 * accumulates sum_t (p_t s4) c + sum_t p_t z4).
 */
typedef struct kvq_decode_int4v_args {
    kvq_decode_args base;
    const uint8_t* v_packed;
    const float* v_scales4;
    const float* v_zeros4;
    int32_t v_group;
} kvq_decode_int4v_args;

kvq_status kvq_decode_attention_int4v(const kvq_decode_int4v_args* a, kvq_stream_t stream);
size_t kvq_decode_int4v_workspace_bytes(const kvq_decode_int4v_args* a);

/*
 * Attention-sink eviction ("Q-TensorFormer" model card, section 6, Attention-Sink
 * Dynamic Eviction): once the context outgrows the memory budget, the cache keeps the
 * first |K_sink| tokens (the sinks) and the tokens with the largest attention mass,
 * the probability alpha_{h,i,j} that query head h gave token j at decode step i,
 * summed over heads and steps.  Three calls make it: a decode step that also adds its
 * mass to a running sum, the selection of the tokens to keep, and the compaction of
 * each cache array to them.  Readings: the mass is kept per batch row (summed over
 * all query heads); equal masses are ordered by the smaller token index; kept tokens
 * keep their relative order.
 *
 * kvq_decode_attention_mass -- kvq_decode_attention (same results) plus
 *   attn_mass[b][t] += sum_h p[b][h][t],  p[b][h][t] = 2^(s[b][h][t] * sm_scale * log2(e) - M) / L,
 * s the step's scores, M and L that head's softmax max (log2 domain) and sum.
 *   base:      as kvq_decode_attention, with base.out required (the merge of the partial
 *              results yields M and L).  base.scores_out may be NULL: the scores then
 *              go to the workspace.
 *   attn_mass: [batch][seq_len] fp32, 4-byte aligned, read and written (start it at 0).
 * Workspace from kvq_decode_mass_workspace_bytes.  Three launches (four with QJL keys:
 * the query sketch); errors as kvq_decode_attention, KVQ_ERR_INVALID_ARG for a missing
 * base.out or attn_mass.
 */
typedef struct kvq_decode_mass_args {
    kvq_decode_args base;
    float* attn_mass;
} kvq_decode_mass_args;

kvq_status kvq_decode_attention_mass(const kvq_decode_mass_args* a, kvq_stream_t stream);
size_t kvq_decode_mass_workspace_bytes(const kvq_decode_mass_args* a);

/*
 * kvq_evict_select -- the tokens a batch row keeps.
 *   mass: [batch][seq_len] fp32 (no NaN), device; kept: [batch][n_keep] int32, device,
 *   written with: tokens 0 .. n_sink-1, then the n_keep - n_sink tokens t >= n_sink of
 *   largest mass[b][t] (equal values, -0 and +0 included: the smaller t first), all in
 *   increasing token order.  Exact: the comparison is on the fp32 values.
 * 0 <= n_sink <= n_keep <= seq_len < 2^31, batch <= 2^31 - 1 (else KVQ_ERR_INVALID_ARG);
 * mass and kept 4-byte aligned.  batch == 0 or n_keep == 0: no launch.  One launch,
 * one CTA per batch row.
 */
kvq_status kvq_evict_select(const float* mass, int64_t batch, int64_t seq_len, int64_t n_sink, int64_t n_keep,
                            int32_t* kept, kvq_stream_t stream);

/*
 * kvq_gather_rows -- compacts one cache array to the kept tokens:
 *   dst[b][h][j][:] = src[b][h][kept[b][j]][:],  j < n_keep,
 * src: [batch][n_heads][src_rows][row_bytes] bytes, dst: [batch][n_heads][dst_rows]
 * [row_bytes] (n_keep <= dst_rows; rows from n_keep on are left as they are), kept:
 * [batch][n_keep] int32 (as kvq_evict_select writes it).  Works on any per-token array
 * of the cache: codes (row_bytes = head_dim), per-token scales (4), sign words
 * (sketch_dim / 8), norms (2), INT4 groups.  src and dst must not overlap (the
 * compaction is not in place).  A kept index outside [0, src_rows) skips that row and
 * records code 0x301 for kvq_device_error.
 * batch, n_heads, n_keep >= 0, row_bytes >= 1, src_rows >= 1 and dst_rows >= n_keep,
 * n_keep * row_bytes < 2^31 (else KVQ_ERR_INVALID_ARG).  Any alignment (the widest
 * access that divides row_bytes and both addresses is used).  One launch.
 */
kvq_status kvq_gather_rows(const void* src, void* dst, int64_t batch, int64_t n_heads, int64_t src_rows,
                           int64_t dst_rows, int64_t row_bytes, const int32_t* kept, int64_t n_keep,
                           kvq_stream_t stream);

/*
 * kvq_gather_rows_multi -- kvq_gather_rows for up to 8 arrays of the same cache (for
 * example K codes, K scales, V codes, V scales) in one launch, all compacted to the
 * same kept tokens.  arrays[i] gives src, dst, src_rows, dst_rows and row_bytes of one
 * array, with the rules of kvq_gather_rows for each (the array list itself is read on
 * the host before the launch).  n_arrays in 1..8 (else KVQ_ERR_INVALID_ARG; 0 with
 * nothing to do: KVQ_OK).  A bad kept index: code 0x301 as kvq_gather_rows.
 */
typedef struct kvq_gather_array {
    const void* src;
    void* dst;
    int64_t src_rows;
    int64_t dst_rows;
    int64_t row_bytes;
} kvq_gather_array;

kvq_status kvq_gather_rows_multi(const kvq_gather_array* arrays, int32_t n_arrays, int64_t batch, int64_t n_heads,
                                 const int32_t* kept, int64_t n_keep, kvq_stream_t stream);

/*
 * kvq_decode_attention_qjlres -- the decode step of kvq_decode_attention over keys
 * stored by kvq_qjl_residual_encode (group-wise INT4 + the 1-bit QJL sketch of the INT4
 * residual), INT8 values.  Per cached token t and query head h (KV head h / G):
 *   score = sum_g s_g * sum_{j in g} q_j c_j + z_g * sum_{j in g} q_j          (<q, k_hat>)
 *           + sqrt(pi/2)/m * ||r||_fp16 * sum_i (S q)_i (2 b_i - 1),          (residual)
 * the INT4 part in fp32 in that factored form, the residual part with the fp32 query
 * sketch (kvq_qjl_query_sketch) through per-CTA byte tables; then softmax and the
 * INT8-value sum exactly as kvq_decode_attention.
 *   base:      key_format = KVQ_KEYS_QJL with k_words / k_norms_f16 = the residual's
 *              sign words and fp16 norms, sketch_f16 / sketch_dim = S and m (128 or
 *              256, else KVQ_ERR_UNSUPPORTED); everything else as kvq_decode_attention
 *              (any group size G = Hq / Hkv).
 *   k_packed4: [B][Hkv][T][D/2] INT4 codes (16-byte aligned); k_scales4, k_zeros4:
 *              [B][Hkv][T][D/k_group] fp32 (4-byte aligned); k_group 32, 64 or 128.
 * Workspace from kvq_decode_qjlres_workspace_bytes.  Errors as kvq_decode_attention.
 */
typedef struct kvq_decode_qjlres_args {
    kvq_decode_args base;
    const uint8_t* k_packed4;
    const float* k_scales4;
    const float* k_zeros4;
    int32_t k_group;
} kvq_decode_qjlres_args;

kvq_status kvq_decode_attention_qjlres(const kvq_decode_qjlres_args* a, kvq_stream_t stream);
size_t kvq_decode_qjlres_workspace_bytes(const kvq_decode_qjlres_args* a);

/*
 * kvq_decode_attention_noalloc -- kvq_decode_attention for callers that cannot
 * allocate device memory and cannot lend a workspace (for example code inside a host
 * engine that has already reserved all device memory through its own allocator, or a
 * latency-critical path where an allocation, which may synchronise the device, is
 * not allowed).  No passage on the pages corresponds to it: it is a deployment
 * variant of the decode step above, with identical arguments and results, except
 * that a->workspace and a->workspace_bytes are ignored.
 *   Scratch: a fixed array of kvq_decode_noalloc_max_workspace_bytes() bytes (8 MiB)
 *   inside the library's device image; every GPU that loads the library keeps it until
 *   the process exits.  A request needing more than that (see
 *   kvq_decode_workspace_bytes) returns KVQ_ERR_WORKSPACE and launches nothing.
 *   The first call on each device looks up the array's device address (a host-side
 *   runtime call, no allocation); make that first call before any stream capture.
 *   All calls share the one array and nothing in it needs to start at zero (every
 *   value read is written earlier in the same call), but calls whose kernels overlap
 *   on the GPU (different streams, or several host threads) race on it: serialise
 *   them.  It calls no cudaMalloc, cudaFree or other allocating routine.
 */
kvq_status kvq_decode_attention_noalloc(const kvq_decode_args* a, kvq_stream_t stream);
size_t kvq_decode_noalloc_max_workspace_bytes(void);

/*
 * kvq_device_error -- read and clear the library's device-side error word on the
 * current device (synchronous: it waits for the device).  Kernels that wait on
 * barriers give up after a bounded number of polls instead of hanging; when they do,
 * they record a nonzero code here and skip the rest of their work.  *code = 0 means
 * no error was recorded.  Returns KVQ_ERR_CUDA if the read itself fails.
 */
kvq_status kvq_device_error(uint32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
