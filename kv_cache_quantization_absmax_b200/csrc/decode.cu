// One decode step over a compressed KV cache: scores -> softmax -> weighted sum of
// INT8 values, for one query token per query head.
//
// Definitions: "GPU-Accelerated INT8 Quantization for KV Cache Compression in Large
// Language Models", abstract (attention scores over the INT8 cache); "QJL: 1-Bit
// Quantized JL Transform for KV Cache Quantization with Zero Overhead", abstract (the
// asymmetric estimator: the query's unquantized JL sketch against the key's sign bits);
// "Q-TensorFormer" model card, section 4 (GQA: query head h reads KV head h / G).
//
// Parallelisation (ours; the pages do not say how decode is parallelised): the T
// cached tokens of each (batch, KV head) unit are cut into `splits` chunks; one CTA per
// (chunk, unit) streams its chunk once and serves all G query heads of the group, so
// each K/V byte is read from HBM exactly once.  It keeps an online-softmax state
// (running max m, running sum l, acc[D]) per head in the base-2 domain and writes it to
// the workspace; a second kernel merges the splits.  No kernel waits on another.
//
// Within a CTA, 8 lanes share a token: for INT8 keys lane j owns dims 16j..16j+15 of
// K and V; for QJL keys lane j owns sign word j (coordinates 32j..32j+31) and dims
// 16j..16j+15 of V.  Codes become floats exactly through the 1.5 * 2^23 bias trick.
//
// QJL scoring uses per-head byte tables built once per CTA in shared memory:
//   LUT[g][b][p] = sum_{k<8} v_g[8p + k] * (bit k of b ? +1 : -1),
// so sum_i v_i (2 b_i - 1) over m = 256 coordinates is 32 table lookups.  The table is
// laid out with the byte position p fastest (32 floats per byte value), and lane
// (sub = j, token group tg) reads byte (e + tg) mod 4 of its word at step e: the 32
// lanes of a warp then read 32 different positions p, i.e. 32 different banks.
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kCodeMagic = 12583040.0f;  // 1.5 * 2^23 + 128
constexpr int kLutP = 32;                  // byte positions per table row (m <= 256)

struct DecodeParams {
    const uint16_t* q;
    const int8_t* kc;
    const float* ks;
    const uint32_t* kw;
    const uint16_t* kn;
    const int8_t* vc;
    const float* vs;
    const float* sketch_v;  // [B * Hq][m] fp32 (QJL)
    float* scores_out;
    float* ws_ml;           // [units * G][splits][2]
    float* ws_acc;          // [units * G][splits][D]
    int64_t T;
    int64_t chunk;
    int Hq;
    int Hkv;
    int splits;
    int m;
    float scale_log2;       // sm_scale * log2(e)
    float qjl_c;            // sqrt(pi/2) / m
    int want_out;
};

// 16 int8 codes (one uint4) -> 16 exact floats.
__device__ __forceinline__ void codes16(const uint4& v, float* c) {
    const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u,
                           v.w ^ 0x80808080u};
#pragma unroll
    for (int i = 0; i < 16; ++i)
        c[i] = __fsub_rn(__uint_as_float(__byte_perm(w[i >> 2], 0x4B400000u, 0x7650u + (i & 3))),
                         kCodeMagic);
}

template <int KEYFMT, int G, int THREADS>
__global__ void __launch_bounds__(THREADS)
decode_partial_kernel(const DecodeParams p) {
    extern __shared__ float dsmem[];
    constexpr int WARPS = THREADS / 32;
    constexpr int TOK_PER_STEP = WARPS * 4;
    const int64_t unit = blockIdx.x;
    const int split = blockIdx.y;
    const int64_t b = unit / p.Hkv;
    const int kvh = (int)(unit % p.Hkv);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tg = lane >> 3;
    const int sub = lane & 7;
    const int64_t T = p.T;
    const int64_t t_begin = (int64_t)split * p.chunk;
    const int64_t t_end = min(T, t_begin + p.chunk);
    const int64_t row0 = unit * T;  // first token row of this unit
    const int nw = p.m / 32;

    // ---- per-lane query slice (INT8) or the byte tables (QJL) ----
    float qv[KEYFMT == KVQ_KEYS_INT8 ? G : 1][16];
    float* lut = dsmem;  // [G][256][kLutP]
    if constexpr (KEYFMT == KVQ_KEYS_INT8) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int64_t h = (int64_t)kvh * G + g;
            const uint4* src = reinterpret_cast<const uint4*>(p.q + (b * p.Hq + h) * kD + sub * 16);
            const uint4 a = __ldg(src), c = __ldg(src + 1);
            const __half2* ha = reinterpret_cast<const __half2*>(&a);
            const __half2* hc = reinterpret_cast<const __half2*>(&c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f0 = __half22float2(ha[i]);
                const float2 f1 = __half22float2(hc[i]);
                qv[g][2 * i] = f0.x;
                qv[g][2 * i + 1] = f0.y;
                qv[g][8 + 2 * i] = f1.x;
                qv[g][8 + 2 * i + 1] = f1.y;
            }
        }
    } else {
        const int npos = p.m / 8;
        for (int idx = threadIdx.x; idx < G * 256 * kLutP; idx += THREADS) {
            const int pos = idx % kLutP;
            const int byte = (idx / kLutP) % 256;
            const int g = idx / (kLutP * 256);
            float acc = 0.0f;
            if (pos < npos) {
                const float* v = p.sketch_v + (b * p.Hq + (int64_t)kvh * G + g) * p.m + pos * 8;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float vk = __ldg(v + k);
                    acc += ((byte >> k) & 1) ? vk : -vk;
                }
            }
            lut[idx] = acc;
        }
        __syncthreads();
    }

    float mrun[G], lrun[G], acc[G][16];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        mrun[g] = -INFINITY;
        lrun[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[g][i] = 0.0f;
    }

    for (int64_t t0 = t_begin; t0 < t_end; t0 += TOK_PER_STEP) {
        const int64_t t = t0 + warp * 4 + tg;
        const bool valid = t < t_end;
        const int64_t r = row0 + (valid ? t : t_begin);
        // ---- scores for the G heads ----
        float score[G];
        if constexpr (KEYFMT == KVQ_KEYS_INT8) {
            const uint4 kv = __ldcs(reinterpret_cast<const uint4*>(p.kc + r * kD) + sub);
            const float ksc = __ldcs(p.ks + r);
            float c[16];
            codes16(kv, c);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float d = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) d = __fmaf_rn(qv[g][i], c[i], d);
                d += __shfl_xor_sync(0xffffffffu, d, 1);
                d += __shfl_xor_sync(0xffffffffu, d, 2);
                d += __shfl_xor_sync(0xffffffffu, d, 4);
                score[g] = d * ksc;
            }
        } else {
            const uint32_t w = sub < nw ? __ldcs(p.kw + r * nw + sub) : 0u;
            const float nrm = __half2float(__ushort_as_half(__ldcs(p.kn + r)));
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float s = 0.0f;
                if (sub < nw) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int byte_sel = (e + tg) & 3;
                        const uint32_t bv = (w >> (8 * byte_sel)) & 0xFFu;
                        s += lut[(g * 256 + (int)bv) * kLutP + sub * 4 + byte_sel];
                    }
                }
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                s += __shfl_xor_sync(0xffffffffu, s, 4);
                score[g] = p.qjl_c * nrm * s;
            }
        }
        if (p.scores_out != nullptr && valid && sub == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g)
                p.scores_out[(b * p.Hq + (int64_t)kvh * G + g) * T + t] = score[g];
        }
        if (!p.want_out || !valid) continue;
        // ---- online softmax + value accumulation ----
        const uint4 vv = __ldcs(reinterpret_cast<const uint4*>(p.vc + r * kD) + sub);
        const float vsc = __ldcs(p.vs + r);
        float c[16];
        codes16(vv, c);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float lg = score[g] * p.scale_log2;
            if (lg > mrun[g]) {
                const float corr = exp2f(mrun[g] - lg);
                lrun[g] *= corr;
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[g][i] *= corr;
                mrun[g] = lg;
            }
            const float pe = exp2f(lg - mrun[g]);
            lrun[g] += pe;
            const float wv = pe * vsc;
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[g][i] = __fmaf_rn(wv, c[i], acc[g][i]);
        }
    }
    if (!p.want_out) return;

    // ---- merge the 4 token groups of each warp (lanes l, l^8, l^16, l^24) ----
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mo = __shfl_xor_sync(0xffffffffu, mrun[g], off);
            const float lo = __shfl_xor_sync(0xffffffffu, lrun[g], off);
            const float mn = fmaxf(mrun[g], mo);
            const float f1 = mn == -INFINITY ? 0.0f : exp2f(mrun[g] - mn);
            const float f2 = mn == -INFINITY ? 0.0f : exp2f(mo - mn);
            lrun[g] = lrun[g] * f1 + lo * f2;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float ao = __shfl_xor_sync(0xffffffffu, acc[g][i], off);
                acc[g][i] = acc[g][i] * f1 + ao * f2;
            }
            mrun[g] = mn;
        }
    }
    // ---- merge the warps through shared memory ----
    __syncthreads();  // the byte tables (QJL) are no longer needed
    float* red_ml = dsmem;                       // [WARPS][G][2]
    float* red_acc = dsmem + WARPS * G * 2;      // [WARPS][G][kD]
    if (tg == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (sub == 0) {
                red_ml[(warp * G + g) * 2] = mrun[g];
                red_ml[(warp * G + g) * 2 + 1] = lrun[g];
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) red_acc[(warp * G + g) * kD + sub * 16 + i] = acc[g][i];
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * kD; idx += THREADS) {
        const int g = idx / kD;
        const int d = idx % kD;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) mx = fmaxf(mx, red_ml[(w * G + g) * 2]);
        float l = 0.0f, a = 0.0f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float mw = red_ml[(w * G + g) * 2];
            const float f = mx == -INFINITY ? 0.0f : exp2f(mw - mx);
            l += red_ml[(w * G + g) * 2 + 1] * f;
            a += red_acc[(w * G + g) * kD + d] * f;
        }
        const int64_t slot = (unit * G + g) * p.splits + split;
        p.ws_acc[slot * kD + d] = a;
        if (d == 0) {
            p.ws_ml[slot * 2] = mx;
            p.ws_ml[slot * 2 + 1] = l;
        }
    }
}

// out[b][h][d] = sum_s acc_s[d] 2^(m_s - M) / sum_s l_s 2^(m_s - M).
__global__ void __launch_bounds__(kD)
decode_combine_kernel(const float* __restrict__ ws_ml, const float* __restrict__ ws_acc, int Hq,
                      int Hkv, int splits, float* __restrict__ out) {
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / Hq;
    const int h = (int)(bh % Hq);
    const int G = Hq / Hkv;
    const int64_t unit = b * Hkv + h / G;
    const int64_t slot0 = (unit * G + (h % G)) * splits;
    const int d = threadIdx.x;
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, ws_ml[(slot0 + s) * 2]);
    float l = 0.0f, a = 0.0f;
    for (int s = 0; s < splits; ++s) {
        const float f = exp2f(ws_ml[(slot0 + s) * 2] - mx);
        l += ws_ml[(slot0 + s) * 2 + 1] * f;
        a += ws_acc[(slot0 + s) * kD + d] * f;
    }
    out[bh * kD + d] = a / l;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kInt8Threads = 128;
constexpr int kQjlThreads = 512;

template <int KEYFMT, int G>
cudaError_t run_partial(const DecodeParams& p, int64_t units, cudaStream_t st) {
    constexpr int THREADS = KEYFMT == KVQ_KEYS_INT8 ? kInt8Threads : kQjlThreads;
    constexpr int WARPS = THREADS / 32;
    size_t smem = (size_t)(WARPS * G * 2 + WARPS * G * kD) * sizeof(float);
    if (KEYFMT == KVQ_KEYS_QJL) {
        const size_t lut = (size_t)G * 256 * kLutP * sizeof(float);
        if (lut > smem) smem = lut;
    }
    auto kern = decode_partial_kernel<KEYFMT, G, THREADS>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)units, (unsigned)p.splits);
    kern<<<grid, THREADS, smem, st>>>(p);
    return cudaGetLastError();
}

template <int KEYFMT>
cudaError_t run_partial_g(int G, const DecodeParams& p, int64_t units, cudaStream_t st) {
    switch (G) {
        case 1: return run_partial<KEYFMT, 1>(p, units, st);
        case 2: return run_partial<KEYFMT, 2>(p, units, st);
        case 4: return run_partial<KEYFMT, 4>(p, units, st);
        case 8:
            if constexpr (KEYFMT == KVQ_KEYS_INT8) return run_partial<KEYFMT, 8>(p, units, st);
            return cudaErrorNotSupported;
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

DecodePlan plan_decode(const kvq_decode_args* a, int sm_count) {
    DecodePlan pl{};
    const int64_t G = a->n_q_heads / a->n_kv_heads;
    pl.units = a->batch * a->n_kv_heads;
    const int64_t T = a->seq_len;
    const bool qjl = a->key_format == KVQ_KEYS_QJL;
    const int64_t target = (int64_t)sm_count * (qjl ? 2 : 16);
    int64_t splits = pl.units > 0 ? (target + pl.units - 1) / pl.units : 1;
    const int64_t min_chunk = qjl ? 1024 : 64;
    int64_t max_splits = (T + min_chunk - 1) / min_chunk;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    int64_t chunk = (T + splits - 1) / splits;
    chunk = (chunk + 15) / 16 * 16;
    splits = (T + chunk - 1) / chunk;
    pl.splits = (int)splits;
    pl.chunk = chunk;
    const int64_t slots = pl.units * G * splits;
    pl.partial_bytes = align256((size_t)slots * 2 * sizeof(float)) +
                       align256((size_t)slots * kD * sizeof(float));
    pl.sketch_bytes = qjl ? align256((size_t)a->batch * a->n_q_heads * a->sketch_dim * sizeof(float)) : 0;
    pl.total_bytes = pl.partial_bytes + pl.sketch_bytes;
    return pl;
}

cudaError_t launch_decode(const kvq_decode_args* a, const DecodePlan& pl, cudaStream_t st) {
    const int G = (int)(a->n_q_heads / a->n_kv_heads);
    const bool qjl = a->key_format == KVQ_KEYS_QJL;
    const int64_t slots = pl.units * G * pl.splits;
    char* ws = static_cast<char*>(a->workspace);
    DecodeParams p{};
    p.q = a->q_f16;
    p.kc = a->k_codes;
    p.ks = a->k_scales;
    p.kw = a->k_words;
    p.kn = a->k_norms_f16;
    p.vc = a->v_codes;
    p.vs = a->v_scales;
    p.scores_out = a->scores_out;
    p.ws_ml = reinterpret_cast<float*>(ws);
    p.ws_acc = reinterpret_cast<float*>(ws + align256((size_t)slots * 2 * sizeof(float)));
    p.sketch_v = qjl ? reinterpret_cast<float*>(ws + pl.partial_bytes) : nullptr;
    p.T = a->seq_len;
    p.chunk = pl.chunk;
    p.Hq = (int)a->n_q_heads;
    p.Hkv = (int)a->n_kv_heads;
    p.splits = pl.splits;
    p.m = qjl ? a->sketch_dim : 0;
    const float sm = a->sm_scale != 0.0f ? a->sm_scale : 1.0f / sqrtf((float)a->head_dim);
    p.scale_log2 = sm * kLog2e;
    p.qjl_c = qjl ? (float)(1.2533141373155002512 / (double)a->sketch_dim) : 0.0f;  // sqrt(pi/2)/m
    p.want_out = a->out != nullptr;
    cudaError_t e;
    if (qjl) {
        e = launch_qjl_query_sketch(a->q_f16, a->batch * a->n_q_heads, a->sketch_f16, a->sketch_dim,
                                    const_cast<float*>(p.sketch_v), st);
        if (e != cudaSuccess) return e;
        e = run_partial_g<KVQ_KEYS_QJL>(G, p, pl.units, st);
    } else {
        e = run_partial_g<KVQ_KEYS_INT8>(G, p, pl.units, st);
    }
    if (e != cudaSuccess || !a->out) return e;
    decode_combine_kernel<<<(unsigned)(a->batch * a->n_q_heads), kD, 0, st>>>(
        p.ws_ml, p.ws_acc, p.Hq, p.Hkv, pl.splits, a->out);
    return cudaGetLastError();
}

}  // namespace kvq
