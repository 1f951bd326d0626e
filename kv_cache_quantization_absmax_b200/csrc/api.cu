// The C ABI (include/kvq.h): host-side argument validation, then dispatch to the
// kernels.  Nothing here allocates device memory or synchronises a stream.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"
#include "kvq_internal.h"

#define KVQ_API extern "C" __attribute__((visibility("default")))

namespace kvq {

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < 64) cached[dev] = n;
    return n;
}

}  // namespace kvq

namespace {

inline bool aligned(const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}
inline bool valid_dtype(int t) { return t == KVQ_F32 || t == KVQ_F16; }
inline kvq_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return KVQ_OK;
    if (e == cudaErrorNotSupported) return KVQ_ERR_UNSUPPORTED;
    return KVQ_ERR_CUDA;
}
inline cudaStream_t cs(kvq_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

constexpr int64_t kMaxQuantDim = 65536;
constexpr int64_t kMaxScoreDim = 8192;

bool qjl_dims_ok(int32_t d, int32_t m) {
    return d == 128 && m >= 32 && m <= 256 && (m % 32) == 0;
}

// Validation shared by kvq_decode_attention and kvq_decode_workspace_bytes.
kvq_status check_decode(const kvq_decode_args* a) {
    if (!a) return KVQ_ERR_INVALID_ARG;
    if (a->batch < 0 || a->n_q_heads <= 0 || a->n_kv_heads <= 0 || a->seq_len <= 0)
        return KVQ_ERR_INVALID_ARG;
    if (a->n_q_heads % a->n_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
    if (a->key_format != KVQ_KEYS_INT8 && a->key_format != KVQ_KEYS_QJL) return KVQ_ERR_INVALID_ARG;
    if (a->head_dim <= 0 || a->head_dim % 16 != 0) return KVQ_ERR_INVALID_ARG;
    if (a->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
    if (!a->out && !a->scores_out) return KVQ_ERR_INVALID_ARG;
    if (!(a->sm_scale == a->sm_scale) || a->sm_scale < 0.0f) return KVQ_ERR_INVALID_ARG;
    if ((a->flags & ~(KVQ_DECODE_CUDA_CORES | KVQ_DECODE_TEST_EXPIRE)) != 0u) return KVQ_ERR_INVALID_ARG;
    if (a->batch == 0) return KVQ_OK;
    if (!a->q_f16 || !aligned(a->q_f16, 16)) return KVQ_ERR_INVALID_ARG;
    if (a->key_format == KVQ_KEYS_INT8) {
        if (!a->k_codes || !a->k_scales || !aligned(a->k_codes, 16) || !aligned(a->k_scales, 4))
            return KVQ_ERR_INVALID_ARG;
    } else {
        if (a->sketch_dim <= 0 || a->sketch_dim % 32 != 0) return KVQ_ERR_INVALID_ARG;
        if (!qjl_dims_ok(a->head_dim, a->sketch_dim)) return KVQ_ERR_UNSUPPORTED;
        if (!a->k_words || !a->k_norms_f16 || !a->sketch_f16) return KVQ_ERR_INVALID_ARG;
        const uintptr_t wa = ((a->sketch_dim / 32) % 4 == 0) ? 16 : 4;
        if (!aligned(a->k_words, wa) || !aligned(a->k_norms_f16, 2) || !aligned(a->sketch_f16, 16))
            return KVQ_ERR_INVALID_ARG;
    }
    if (a->out) {
        if (!a->v_codes || !a->v_scales || !aligned(a->v_codes, 16) || !aligned(a->v_scales, 4) ||
            !aligned(a->out, 16))
            return KVQ_ERR_INVALID_ARG;
    }
    if (a->scores_out && !aligned(a->scores_out, 4)) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

}  // namespace

KVQ_API int kvq_abi_version(void) { return KVQ_ABI_VERSION; }

KVQ_API const char* kvq_status_string(kvq_status s) {
    switch (s) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_INVALID_ARG: return "invalid argument";
        case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
        case KVQ_ERR_CUDA: return "CUDA runtime error";
        case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
        case KVQ_ERR_DEVICE: return "device-side error recorded";
    }
    return "unknown status";
}

KVQ_API kvq_status kvq_quantize_int8(const void* x, kvq_dtype x_dtype, int64_t n_rows, int64_t d,
                                     int8_t* codes, float* scales, kvq_stream_t stream) {
    if (!valid_dtype(x_dtype) || n_rows < 0 || d <= 0 || d % 16 != 0 || d > kMaxQuantDim)
        return KVQ_ERR_INVALID_ARG;
    if (n_rows == 0) return KVQ_OK;
    if (!x || !codes || !scales || !aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_quantize_int8(x, x_dtype == KVQ_F16, n_rows, d, codes, scales,
                                               cs(stream)));
}

KVQ_API kvq_status kvq_dequantize_int8(const int8_t* codes, const float* scales, int64_t n_rows,
                                       int64_t d, void* out, kvq_dtype out_dtype,
                                       kvq_stream_t stream) {
    if (!valid_dtype(out_dtype) || n_rows < 0 || d <= 0 || d % 16 != 0) return KVQ_ERR_INVALID_ARG;
    if (n_rows == 0) return KVQ_OK;
    if (!codes || !scales || !out || !aligned(codes, 16) || !aligned(scales, 4) || !aligned(out, 16))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_dequantize_int8(codes, scales, n_rows, d, out,
                                                 out_dtype == KVQ_F16, cs(stream)));
}

KVQ_API kvq_status kvq_int8_scores(const void* q, kvq_dtype q_dtype, const int8_t* codes,
                                   const float* scales, int64_t n_rows, int64_t d, float* scores,
                                   kvq_stream_t stream) {
    if (!valid_dtype(q_dtype) || n_rows < 0 || d <= 0 || d % 16 != 0 || d > kMaxScoreDim)
        return KVQ_ERR_INVALID_ARG;
    if (n_rows == 0) return KVQ_OK;
    if (!q || !codes || !scales || !scores || !aligned(q, 16) || !aligned(codes, 16) ||
        !aligned(scales, 4) || !aligned(scores, 4))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_int8_scores(q, q_dtype == KVQ_F16, codes, scales, n_rows, d,
                                             scores, cs(stream)));
}

KVQ_API kvq_status kvq_qjl_encode(const uint16_t* keys_f16, int64_t n_keys, int32_t d,
                                  const uint16_t* sketch_f16, int32_t m, uint32_t* sign_words,
                                  uint16_t* norms_f16, kvq_stream_t stream) {
    if (n_keys < 0 || d <= 0 || d % 16 != 0 || m <= 0 || m % 32 != 0) return KVQ_ERR_INVALID_ARG;
    if (!qjl_dims_ok(d, m)) return KVQ_ERR_UNSUPPORTED;
    if (n_keys == 0) return KVQ_OK;
    const uintptr_t wa = ((m / 32) % 4 == 0) ? 16 : 4;
    if (!keys_f16 || !sketch_f16 || !sign_words || !norms_f16 || !aligned(keys_f16, 16) ||
        !aligned(sketch_f16, 16) || !aligned(sign_words, wa) || !aligned(norms_f16, 2))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_qjl_encode(keys_f16, n_keys, sketch_f16, m, sign_words, norms_f16,
                                            cs(stream)));
}

KVQ_API kvq_status kvq_qjl_query_sketch(const uint16_t* q_f16, int64_t n_q, int32_t d,
                                        const uint16_t* sketch_f16, int32_t m, float* v,
                                        kvq_stream_t stream) {
    if (n_q < 0 || d <= 0 || d % 16 != 0 || m <= 0 || m % 32 != 0) return KVQ_ERR_INVALID_ARG;
    if (!qjl_dims_ok(d, m)) return KVQ_ERR_UNSUPPORTED;
    if (n_q == 0) return KVQ_OK;
    if (!q_f16 || !sketch_f16 || !v || !aligned(q_f16, 16) || !aligned(sketch_f16, 16) ||
        !aligned(v, 16))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_qjl_query_sketch(q_f16, n_q, sketch_f16, m, v, cs(stream)));
}

KVQ_API kvq_status kvq_quantize_int8_channelwise(const void* x, kvq_dtype x_dtype, int64_t n_blocks,
                                                 int64_t rows, int64_t d, int8_t* codes, float* scales,
                                                 kvq_stream_t stream) {
    if (!valid_dtype(x_dtype) || n_blocks < 0 || rows <= 0 || d <= 0 || d % 64 != 0)
        return KVQ_ERR_INVALID_ARG;
    if (n_blocks == 0) return KVQ_OK;
    if (n_blocks > 65535) return KVQ_ERR_UNSUPPORTED;
    if (!x || !codes || !scales || !aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_quantize_int8_channelwise(x, x_dtype == KVQ_F16, n_blocks, rows, d,
                                                           codes, scales, cs(stream)));
}

KVQ_API kvq_status kvq_dequantize_int8_channelwise(const int8_t* codes, const float* scales, int64_t n_blocks,
                                                   int64_t rows, int64_t d, void* out, kvq_dtype out_dtype,
                                                   kvq_stream_t stream) {
    if (!valid_dtype(out_dtype) || n_blocks < 0 || rows <= 0 || d <= 0 || d % 64 != 0)
        return KVQ_ERR_INVALID_ARG;
    if (n_blocks == 0) return KVQ_OK;
    if (n_blocks > 65535 || rows * d >= (int64_t(1) << 35)) return KVQ_ERR_UNSUPPORTED;
    if (!codes || !scales || !out || !aligned(codes, 16) || !aligned(scales, 4) || !aligned(out, 16))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_dequantize_int8_channelwise(codes, scales, n_blocks, rows, d, out,
                                                             out_dtype == KVQ_F16, cs(stream)));
}

KVQ_API kvq_status kvq_quantize_int4(const void* x, kvq_dtype x_dtype, int64_t n_rows, int64_t d,
                                     int32_t group, uint8_t* packed, float* scales, float* zeros,
                                     kvq_stream_t stream) {
    if (!valid_dtype(x_dtype) || n_rows < 0 || d <= 0 || group <= 0 || d % group != 0)
        return KVQ_ERR_INVALID_ARG;
    if (group != 32 && group != 64 && group != 128) return KVQ_ERR_UNSUPPORTED;
    if (n_rows == 0) return KVQ_OK;
    if (!x || !packed || !scales || !zeros || !aligned(x, 16) || !aligned(packed, 16) ||
        !aligned(scales, 4) || !aligned(zeros, 4))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_quantize_int4(x, x_dtype == KVQ_F16, n_rows, d, group, packed, scales, zeros,
                                               cs(stream)));
}

KVQ_API kvq_status kvq_qjl_residual_encode(const uint16_t* keys_f16, int64_t n_keys, int32_t d, int32_t group,
                                           const uint16_t* sketch_f16, int32_t m, uint8_t* packed, float* scales,
                                           float* zeros, uint16_t* residual_f16, uint32_t* sign_words,
                                           uint16_t* rnorms_f16, kvq_stream_t stream) {
    if (n_keys < 0 || d <= 0 || d % 16 != 0 || group <= 0 || d % group != 0 || m <= 0 || m % 32 != 0)
        return KVQ_ERR_INVALID_ARG;
    if (group != 32 && group != 64 && group != 128) return KVQ_ERR_UNSUPPORTED;
    if (!qjl_dims_ok(d, m)) return KVQ_ERR_UNSUPPORTED;
    if (n_keys == 0) return KVQ_OK;
    const uintptr_t wa = ((m / 32) % 4 == 0) ? 16 : 4;
    if (!keys_f16 || !sketch_f16 || !packed || !scales || !zeros || !residual_f16 || !sign_words ||
        !rnorms_f16 || !aligned(keys_f16, 16) || !aligned(sketch_f16, 16) || !aligned(packed, 16) ||
        !aligned(scales, 4) || !aligned(zeros, 4) || !aligned(residual_f16, 16) || !aligned(sign_words, wa) ||
        !aligned(rnorms_f16, 2))
        return KVQ_ERR_INVALID_ARG;
    cudaStream_t s = cs(stream);
    const cudaError_t e = kvq::launch_quantize_int4_residual(keys_f16, n_keys, d, group, packed, scales, zeros,
                                                             residual_f16, s);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(kvq::launch_qjl_encode(residual_f16, n_keys, sketch_f16, m, sign_words, rnorms_f16, s));
}

KVQ_API kvq_status kvq_dequantize_int4(const uint8_t* packed, const float* scales, const float* zeros,
                                       int64_t n_rows, int64_t d, int32_t group, void* out,
                                       kvq_dtype out_dtype, kvq_stream_t stream) {
    if (!valid_dtype(out_dtype) || n_rows < 0 || d <= 0 || group <= 0 || d % group != 0)
        return KVQ_ERR_INVALID_ARG;
    if (group != 32 && group != 64 && group != 128) return KVQ_ERR_UNSUPPORTED;
    if (n_rows == 0) return KVQ_OK;
    if (!packed || !scales || !zeros || !out || !aligned(packed, 4) || !aligned(scales, 4) ||
        !aligned(zeros, 4) || !aligned(out, 16))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_dequantize_int4(packed, scales, zeros, n_rows, d, group, out,
                                                 out_dtype == KVQ_F16, cs(stream)));
}

KVQ_API size_t kvq_decode_workspace_bytes(const kvq_decode_args* a) {
    if (check_decode(a) != KVQ_OK) return 0;
    return kvq::plan_decode(a, kvq::device_sm_count()).total_bytes;
}

KVQ_API kvq_status kvq_decode_attention(const kvq_decode_args* a, kvq_stream_t stream) {
    const kvq_status st = check_decode(a);
    if (st != KVQ_OK) return st;
    if (a->batch == 0) return KVQ_OK;
    const kvq::DecodePlan plan = kvq::plan_decode(a, kvq::device_sm_count());
    if (!a->workspace || !aligned(a->workspace, 256) || a->workspace_bytes < plan.total_bytes)
        return KVQ_ERR_WORKSPACE;
    return from_cuda(kvq::launch_decode(a, plan, cs(stream)));
}

namespace {

// The decode arguments of an append call as the kernels see them (T + 1 tokens), after
// validating the append-specific fields.
kvq_status check_append(const kvq_decode_append_args* a, kvq_decode_args* view) {
    if (!a) return KVQ_ERR_INVALID_ARG;
    const int64_t T = a->base.seq_len;
    if (T < 0 || a->capacity < T + 1) return KVQ_ERR_INVALID_ARG;
    *view = a->base;
    view->seq_len = T + 1;
    const kvq_status st = check_decode(view);
    if (st != KVQ_OK || view->batch == 0) return st;
    if (!a->k_new_f16 || !aligned(a->k_new_f16, 16)) return KVQ_ERR_INVALID_ARG;
    if (view->out && (!a->v_new_f16 || !aligned(a->v_new_f16, 16))) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

}  // namespace

KVQ_API size_t kvq_decode_append_workspace_bytes(const kvq_decode_append_args* a) {
    kvq_decode_args view;
    if (check_append(a, &view) != KVQ_OK) return 0;
    return kvq::plan_decode(&view, kvq::device_sm_count()).total_bytes;
}

KVQ_API kvq_status kvq_decode_append(const kvq_decode_append_args* a, kvq_stream_t stream) {
    kvq_decode_args view;
    const kvq_status st = check_append(a, &view);
    if (st != KVQ_OK) return st;
    if (view.batch == 0) return KVQ_OK;
    const kvq::DecodePlan plan = kvq::plan_decode(&view, kvq::device_sm_count());
    if (!view.workspace || !aligned(view.workspace, 256) || view.workspace_bytes < plan.total_bytes)
        return KVQ_ERR_WORKSPACE;
    const kvq::AppendSpec app{a->capacity, a->k_new_f16, a->v_new_f16};
    return from_cuda(kvq::launch_decode(&view, plan, cs(stream), &app));
}

namespace {

// The decode arguments of an INT4-value call as the shared checks see them (the INT4
// arrays stand in for the INT8 value arrays, with the same alignment rules).
kvq_status check_int4v(const kvq_decode_int4v_args* a, kvq_decode_args* view) {
    if (!a) return KVQ_ERR_INVALID_ARG;
    *view = a->base;
    if (view->key_format != KVQ_KEYS_INT8) return KVQ_ERR_UNSUPPORTED;
    if (view->out) {
        view->v_codes = reinterpret_cast<const int8_t*>(a->v_packed);
        view->v_scales = a->v_scales4;
    }
    const kvq_status st = check_decode(view);
    if (st != KVQ_OK || view->batch == 0 || !view->out) return st;
    if (a->v_group != 32 && a->v_group != 64 && a->v_group != 128) return KVQ_ERR_UNSUPPORTED;
    if (!a->v_zeros4 || !aligned(a->v_zeros4, 4)) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

}  // namespace

KVQ_API size_t kvq_decode_int4v_workspace_bytes(const kvq_decode_int4v_args* a) {
    kvq_decode_args view;
    if (check_int4v(a, &view) != KVQ_OK) return 0;
    return kvq::plan_decode(&view, kvq::device_sm_count(), false).total_bytes;
}

KVQ_API kvq_status kvq_decode_attention_int4v(const kvq_decode_int4v_args* a, kvq_stream_t stream) {
    kvq_decode_args view;
    const kvq_status st = check_int4v(a, &view);
    if (st != KVQ_OK) return st;
    if (view.batch == 0) return KVQ_OK;
    const kvq::DecodePlan plan = kvq::plan_decode(&view, kvq::device_sm_count(), false);
    if (!view.workspace || !aligned(view.workspace, 256) || view.workspace_bytes < plan.total_bytes)
        return KVQ_ERR_WORKSPACE;
    const kvq::Int4Values v4{a->v_packed, a->v_scales4, a->v_zeros4, a->v_group};
    return from_cuda(kvq::launch_decode(&view, plan, cs(stream), nullptr, &v4));
}

namespace {

// Workspace of a mass decode: the decode's own, then [B * Hq][2] fp32 final max/sum, then
// (when the caller passes no scores buffer) the [B][Hq][T] fp32 scores.
struct MassLayout {
    kvq::DecodePlan plan;
    size_t ml_off, scores_off, total;
};

MassLayout mass_layout(const kvq_decode_args* a) {
    MassLayout l;
    l.plan = kvq::plan_decode(a, kvq::device_sm_count());
    const auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    l.ml_off = up(l.plan.total_bytes);
    l.scores_off = up(l.ml_off + (size_t)a->batch * a->n_q_heads * 2 * sizeof(float));
    l.total = l.scores_off + (a->scores_out ? 0 : (size_t)a->batch * a->n_q_heads * a->seq_len * sizeof(float));
    return l;
}

kvq_status check_mass(const kvq_decode_mass_args* a) {
    if (!a) return KVQ_ERR_INVALID_ARG;
    if (!a->base.out) return KVQ_ERR_INVALID_ARG;
    const kvq_status st = check_decode(&a->base);
    if (st != KVQ_OK || a->base.batch == 0) return st;
    if (!a->attn_mass || !aligned(a->attn_mass, 4)) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

}  // namespace

KVQ_API size_t kvq_decode_mass_workspace_bytes(const kvq_decode_mass_args* a) {
    if (check_mass(a) != KVQ_OK || a->base.batch == 0) return 0;
    return mass_layout(&a->base).total;
}

KVQ_API kvq_status kvq_decode_attention_mass(const kvq_decode_mass_args* a, kvq_stream_t stream) {
    const kvq_status st = check_mass(a);
    if (st != KVQ_OK) return st;
    if (a->base.batch == 0) return KVQ_OK;
    const MassLayout l = mass_layout(&a->base);
    if (!a->base.workspace || !aligned(a->base.workspace, 256) || a->base.workspace_bytes < l.total)
        return KVQ_ERR_WORKSPACE;
    kvq_decode_args view = a->base;
    char* ws = static_cast<char*>(a->base.workspace);
    float* fin_ml = reinterpret_cast<float*>(ws + l.ml_off);
    if (!view.scores_out) view.scores_out = reinterpret_cast<float*>(ws + l.scores_off);
    cudaStream_t s = cs(stream);
    cudaError_t e = kvq::launch_decode(&view, l.plan, s, nullptr, nullptr, fin_ml);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(kvq::launch_attention_mass(view.scores_out, fin_ml, view.batch, view.n_q_heads,
                                                view.seq_len, kvq::decode_scale_log2(&view), a->attn_mass, s));
}

KVQ_API kvq_status kvq_evict_select(const float* mass, int64_t batch, int64_t seq_len, int64_t n_sink,
                                    int64_t n_keep, int32_t* kept, kvq_stream_t stream) {
    if (batch < 0 || batch > INT32_MAX || n_sink < 0 || n_keep < n_sink || seq_len < n_keep || seq_len > INT32_MAX)
        return KVQ_ERR_INVALID_ARG;
    if (batch == 0 || n_keep == 0) return KVQ_OK;
    if (!mass || !kept || !aligned(mass, 4) || !aligned(kept, 4)) return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_evict_select(mass, batch, seq_len, n_sink, n_keep, kept, cs(stream)));
}

KVQ_API kvq_status kvq_gather_rows(const void* src, void* dst, int64_t batch, int64_t n_heads, int64_t src_rows,
                                   int64_t dst_rows, int64_t row_bytes, const int32_t* kept, int64_t n_keep,
                                   kvq_stream_t stream) {
    if (batch < 0 || n_heads < 0 || n_keep < 0 || row_bytes < 1 || src_rows < 1 || dst_rows < n_keep ||
        n_keep * row_bytes >= ((int64_t)1 << 31) || n_heads > INT32_MAX)
        return KVQ_ERR_INVALID_ARG;
    if (batch == 0 || n_heads == 0 || n_keep == 0) return KVQ_OK;
    if (!src || !dst || !kept || !aligned(kept, 4)) return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_gather_rows(src, dst, batch, n_heads, src_rows, dst_rows, row_bytes, kept, n_keep,
                                             cs(stream)));
}

KVQ_API kvq_status kvq_gather_rows_multi(const kvq_gather_array* arrays, int32_t n_arrays, int64_t batch,
                                         int64_t n_heads, const int32_t* kept, int64_t n_keep, kvq_stream_t stream) {
    if (n_arrays < 0 || n_arrays > 8 || batch < 0 || n_heads < 0 || n_keep < 0 || n_heads > INT32_MAX)
        return KVQ_ERR_INVALID_ARG;
    if (n_arrays > 0 && !arrays) return KVQ_ERR_INVALID_ARG;
    kvq::GatherArray ga[8];
    for (int i = 0; i < n_arrays; ++i) {
        const kvq_gather_array& g = arrays[i];
        if (g.row_bytes < 1 || g.src_rows < 1 || g.dst_rows < n_keep || n_keep * g.row_bytes >= ((int64_t)1 << 31))
            return KVQ_ERR_INVALID_ARG;
        ga[i] = kvq::GatherArray{g.src, g.dst, g.src_rows, g.dst_rows, g.row_bytes};
    }
    if (n_arrays == 0 || batch == 0 || n_heads == 0 || n_keep == 0) return KVQ_OK;
    if (!kept || !aligned(kept, 4)) return KVQ_ERR_INVALID_ARG;
    for (int i = 0; i < n_arrays; ++i)
        if (!ga[i].src || !ga[i].dst) return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_gather_rows_multi(ga, n_arrays, batch, n_heads, kept, n_keep, cs(stream)));
}

namespace {

// Residual keys: the decode arguments carry the residual's sign words, norms and the
// sketch as QJL keys; the INT4 stage comes in the extra fields.
kvq_status check_qjlres(const kvq_decode_qjlres_args* a) {
    if (!a) return KVQ_ERR_INVALID_ARG;
    if (a->base.key_format != KVQ_KEYS_QJL) return KVQ_ERR_INVALID_ARG;
    const kvq_status st = check_decode(&a->base);
    if (st != KVQ_OK) return st;
    if (a->k_group != 32 && a->k_group != 64 && a->k_group != 128) return KVQ_ERR_UNSUPPORTED;
    if (a->base.sketch_dim != 128 && a->base.sketch_dim != 256) return KVQ_ERR_UNSUPPORTED;
    if (a->base.batch == 0) return KVQ_OK;
    if (!a->k_packed4 || !a->k_scales4 || !a->k_zeros4 || !aligned(a->k_packed4, 16) ||
        !aligned(a->k_scales4, 4) || !aligned(a->k_zeros4, 4) || !aligned(a->base.k_words, 16))
        return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

}  // namespace

KVQ_API size_t kvq_decode_qjlres_workspace_bytes(const kvq_decode_qjlres_args* a) {
    if (check_qjlres(a) != KVQ_OK || a->base.batch == 0) return 0;
    return kvq::plan_decode(&a->base, kvq::device_sm_count()).total_bytes;
}

KVQ_API kvq_status kvq_decode_attention_qjlres(const kvq_decode_qjlres_args* a, kvq_stream_t stream) {
    const kvq_status st = check_qjlres(a);
    if (st != KVQ_OK) return st;
    if (a->base.batch == 0) return KVQ_OK;
    const kvq::DecodePlan plan = kvq::plan_decode(&a->base, kvq::device_sm_count());
    if (!a->base.workspace || !aligned(a->base.workspace, 256) || a->base.workspace_bytes < plan.total_bytes)
        return KVQ_ERR_WORKSPACE;
    const kvq::Int4Keys k4{a->k_packed4, a->k_scales4, a->k_zeros4, a->k_group};
    return from_cuda(kvq::launch_decode(&a->base, plan, cs(stream), nullptr, nullptr, nullptr, &k4));
}

KVQ_API kvq_status kvq_device_error(uint32_t* code) {
    if (!code) return KVQ_ERR_INVALID_ARG;
    uint32_t a = 0, b = 0, c = 0;
    if (kvq::read_and_clear_device_error(&a) != cudaSuccess) return KVQ_ERR_CUDA;
    if (kvq::read_and_clear_decode_error(&b) != cudaSuccess) return KVQ_ERR_CUDA;
    if (kvq::read_and_clear_evict_error(&c) != cudaSuccess) return KVQ_ERR_CUDA;
    *code = a ? a : (b ? b : c);
    return KVQ_OK;
}
