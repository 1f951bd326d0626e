// Internal declarations shared by the library's translation units (host side).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

int device_sm_count();  // SM count of the current device (cached per device)

// quantize.cu
cudaError_t launch_quantize_int8(const void* x, bool f16, int64_t n_rows, int64_t d,
                                 int8_t* codes, float* scales, cudaStream_t st);
cudaError_t launch_dequantize_int8(const int8_t* codes, const float* scales, int64_t n_rows,
                                   int64_t d, void* out, bool f16, cudaStream_t st);
cudaError_t launch_int8_scores(const void* q, bool q_f16, const int8_t* codes,
                               const float* scales, int64_t n_rows, int64_t d, float* scores,
                               cudaStream_t st);

// lowbit.cu
cudaError_t launch_quantize_int4(const void* x, bool f16, int64_t n_rows, int64_t d, int group,
                                 uint8_t* packed, float* scales, float* zeros, cudaStream_t st);
cudaError_t launch_quantize_int4_residual(const uint16_t* x, int64_t n_rows, int64_t d, int group,
                                          uint8_t* packed, float* scales, float* zeros, uint16_t* resid,
                                          cudaStream_t st);
cudaError_t launch_dequantize_int4(const uint8_t* packed, const float* scales, const float* zeros,
                                   int64_t n_rows, int64_t d, int group, void* out, bool f16,
                                   cudaStream_t st);
cudaError_t launch_quantize_int8_channelwise(const void* x, bool f16, int64_t n_blocks, int64_t rows,
                                             int64_t d, int8_t* codes, float* scales, cudaStream_t st);
cudaError_t launch_dequantize_int8_channelwise(const int8_t* codes, const float* scales, int64_t n_blocks,
                                               int64_t rows, int64_t d, void* out, bool f16,
                                               cudaStream_t st);

// qjl.cu
// Returns cudaErrorNotSupported when the driver's tensor-map encoder is unavailable.
cudaError_t launch_qjl_encode(const uint16_t* keys, int64_t n_keys, const uint16_t* S, int m,
                              uint32_t* words, uint16_t* norms, cudaStream_t st);
// TMA descriptor of a byte tensor [rows][128] (box 128 bytes x box_rows, 128-byte
// swizzle); false if the driver's encoder is unavailable or rejects the arguments.
bool make_u8_rows_map(CUtensorMap* map, const void* ptr, int64_t rows, int box_rows);
cudaError_t launch_qjl_query_sketch(const uint16_t* q, int64_t n_q, const uint16_t* S, int m,
                                    float* v, cudaStream_t st);
cudaError_t read_and_clear_device_error(uint32_t* code);

// decode.cu
struct DecodePlan {
    int G;                // query heads per CTA (a power of two dividing Hq / Hkv)
    int nsub;             // head subgroups per KV head: (Hq / Hkv) / G
    int64_t units;        // B * Hkv
    int ctas;             // CTAs of the partial kernel: nsub per contiguous token range
    int64_t W;            // tokens per range
    int maxj;             // unit segments one range can touch
    bool int8_tc;         // INT8 keys: the tensor-core kernel, one CTA per SM
    size_t partial_bytes; // per-segment softmax states
    size_t sketch_bytes;  // query sketches (QJL)
    size_t total_bytes;
};
// tc_capable: the call may run the tensor-core INT8 kernel (decodes and appends with INT8
// values; not the INT4-value entry point)
DecodePlan plan_decode(const kvq_decode_args* a, int sm_count, bool tc_capable = true);
cudaError_t read_and_clear_decode_error(uint32_t* code);
// Append-on-decode: the new token (row T - 1 of every unit, a->seq_len = T) is encoded
// by the decode kernel itself; the cache arrays have `capacity` rows per unit.
struct AppendSpec {
    int64_t capacity;
    const uint16_t* k_new;
    const uint16_t* v_new;  // null: values not appended
};
// INT4 values (group-wise, packed): replace a->v_codes / a->v_scales.
struct Int4Values {
    const uint8_t* packed;
    const float* scales;
    const float* zeros;
    int group;
};
// sm_scale * log2(e), the factor the decode kernels apply to a score before exp2.
float decode_scale_log2(const kvq_decode_args* a);
// fin_ml (optional, [B * Hq][2]): each query head's final softmax max (log2 domain) and
// sum, written by the combine kernel (needs a->out).
// Residual keys: group-wise INT4 codes [units * T][D / 2], scales and zero points
// [units * T][D / group]; the residual's sign words and norms come in k_words /
// k_norms_f16 of the decode arguments (key_format QJL).
struct Int4Keys {
    const uint8_t* packed;
    const float* scales;
    const float* zeros;
    int group;
};
cudaError_t launch_decode(const kvq_decode_args* a, const DecodePlan& plan, cudaStream_t st,
                          const AppendSpec* app = nullptr, const Int4Values* v4 = nullptr,
                          float* fin_ml = nullptr, const Int4Keys* k4 = nullptr);

// evict.cu
cudaError_t launch_attention_mass(const float* scores, const float* fin_ml, int64_t B, int64_t Hq,
                                  int64_t T, float scale_log2, float* mass, cudaStream_t st);
cudaError_t launch_evict_select(const float* mass, int64_t B, int64_t T, int64_t n_sink, int64_t n_keep,
                                int32_t* kept, cudaStream_t st);
cudaError_t launch_gather_rows(const void* src, void* dst, int64_t B, int64_t H, int64_t src_rows,
                               int64_t dst_rows, int64_t row_bytes, const int32_t* kept, int64_t n_keep,
                               cudaStream_t st);
struct GatherArray {
    const void* src;
    void* dst;
    int64_t src_rows, dst_rows, row_bytes;
};
cudaError_t launch_gather_rows_multi(const GatherArray* arrays, int n_arrays, int64_t B, int64_t H,
                                     const int32_t* kept, int64_t n_keep, cudaStream_t st);
cudaError_t read_and_clear_evict_error(uint32_t* code);

}  // namespace kvq
