// Per-row absmax INT8 quantize / dequantize and INT8 attention scores.
//
// Definitions: "Q-TensorFormer" model card, section 6, symmetric INT8 equation
// (X_hat = clamp(round(X / s8), -128, 127) * s8, s8 = max|X| / 127), applied per row of
// head_dim; "GPU-Accelerated INT8 Quantization for KV Cache Compression in Large
// Language Models", abstract (attention-score error of the INT8 cache).
//
// All three kernels stream HBM: each element is read once and written once, with
// 16-byte vector accesses whose addresses are contiguous across the lanes of every
// instruction.  Quantize keeps each row in registers between the absmax reduction
// (warp shuffles, plus shared memory for rows wider than a warp) and the code pass.
//
// Bit-exactness of the codes: see kvq_int8.cuh.
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_int8.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

using i8::pack_low_bytes;
using i8::quantize_values;
using i8::scale_reciprocal;

constexpr float kCodeMagic = 12583040.0f;           // 1.5 * 2^23 + 128

template <typename T> struct VecTraits;
template <> struct VecTraits<__half> { static constexpr int kPerVec = 8; };
template <> struct VecTraits<float> { static constexpr int kPerVec = 4; };

__device__ __forceinline__ void unpack(const uint4& v, float* f, __half) {
    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __half22float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ void unpack(const uint4& v, float* f, float) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}

// max |x| over one 16-byte vector (exact: max of magnitudes).
__device__ __forceinline__ float vec_absmax(const uint4& v, __half) {
    const __half2* h = reinterpret_cast<const __half2*>(&v);
    __half2 m = __habs2(h[0]);
    m = __hmax2(m, __habs2(h[1]));
    m = __hmax2(m, __habs2(h[2]));
    m = __hmax2(m, __habs2(h[3]));
    return fmaxf(__low2float(m), __high2float(m));
}
__device__ __forceinline__ float vec_absmax(const uint4& v, float) {
    return fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                 fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
}

template <int BYTES>
__device__ __forceinline__ void store_codes(int8_t* dst, const uint32_t* w) {
    if constexpr (BYTES == 4) {
        *reinterpret_cast<uint32_t*>(dst) = w[0];
    } else if constexpr (BYTES == 8) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    } else {
        static_assert(BYTES == 16, "");
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Rows of D = TPR * VPT * kPerVec elements; TPR (<= 32) lanes share a row; each lane
// holds VPT 16-byte vectors of its row, vector i of lane l at row offset (i * TPR + l)
// so every load instruction covers TPR * 16 contiguous bytes; RPT rows in flight.
template <typename T, int TPR, int VPT, int RPT>
__global__ void __launch_bounds__(256)
quantize_rows_warp(const T* __restrict__ x, int64_t n_rows, int8_t* __restrict__ codes,
                   float* __restrict__ scales) {
    constexpr int PV = VecTraits<T>::kPerVec;
    constexpr int D = TPR * VPT * PV;
    constexpr int GROUPS = 256 / TPR;
    constexpr int ROWS_PER_ITER = GROUPS * RPT;
    const int lane = threadIdx.x % TPR;
    const int group = threadIdx.x / TPR;
    for (int64_t base = (int64_t)blockIdx.x * ROWS_PER_ITER; base < n_rows;
         base += (int64_t)gridDim.x * ROWS_PER_ITER) {
        uint4 v[RPT][VPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int64_t row = base + r * GROUPS + group;
            const uint4* src = reinterpret_cast<const uint4*>(x + row * D);
#pragma unroll
            for (int i = 0; i < VPT; ++i)
                v[r][i] = row < n_rows ? __ldcs(src + i * TPR + lane) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int64_t row = base + r * GROUPS + group;
            float a = 0.0f;
#pragma unroll
            for (int i = 0; i < VPT; ++i) a = fmaxf(a, vec_absmax(v[r][i], T()));
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1)
                a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
            const float s = __fdiv_rn(a, 127.0f);
            const float rinv = scale_reciprocal(s);
            if (row < n_rows) {
                if (lane == 0) scales[row] = s;
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    float f[PV];
                    unpack(v[r][i], f, T());
                    uint32_t w[PV / 4];
                    quantize_values<PV>(f, s, rinv, w);
                    store_codes<PV>(codes + row * D + (int64_t)(i * TPR + lane) * PV, w);
                }
            }
        }
    }
}

// One CTA of 256 threads per row of D = 256 * VPT * kPerVec elements.
template <typename T, int VPT>
__global__ void __launch_bounds__(256)
quantize_rows_cta(const T* __restrict__ x, int64_t n_rows, int8_t* __restrict__ codes,
                  float* __restrict__ scales) {
    constexpr int PV = VecTraits<T>::kPerVec;
    constexpr int D = 256 * VPT * PV;
    __shared__ float red[8];
    const int tid = threadIdx.x;
    for (int64_t row = blockIdx.x; row < n_rows; row += gridDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(x + row * D);
        uint4 v[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) v[i] = __ldcs(src + i * 256 + tid);
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) a = fmaxf(a, vec_absmax(v[i], T()));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        if ((tid & 31) == 0) red[tid >> 5] = a;
        __syncthreads();
        a = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) a = fmaxf(a, red[w]);
        const float s = __fdiv_rn(a, 127.0f);
        const float rinv = scale_reciprocal(s);
        if (tid == 0) scales[row] = s;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            float f[PV];
            unpack(v[i], f, T());
            uint32_t w[PV / 4];
            quantize_values<PV>(f, s, rinv, w);
            store_codes<PV>(codes + row * D + (int64_t)(i * 256 + tid) * PV, w);
        }
        __syncthreads();  // red[] is reused by the next row
    }
}

// Any D that is a multiple of 16: one warp per row, two passes over the row (the second
// pass re-reads it through L1/L2).  Used for widths without a specialised kernel.
template <typename T>
__global__ void __launch_bounds__(256)
quantize_rows_generic(const T* __restrict__ x, int64_t n_rows, int64_t d,
                      int8_t* __restrict__ codes, float* __restrict__ scales) {
    constexpr int PV = VecTraits<T>::kPerVec;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = d / PV;
    for (int64_t row = warp; row < n_rows; row += n_warps) {
        const uint4* src = reinterpret_cast<const uint4*>(x + row * d);
        float a = 0.0f;
        for (int64_t i = lane; i < nvec; i += 32) {
            float f[PV];
            unpack(src[i], f, T());
#pragma unroll
            for (int e = 0; e < PV; ++e) a = fmaxf(a, fabsf(f[e]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        const float s = __fdiv_rn(a, 127.0f);
        const float rinv = scale_reciprocal(s);
        if (lane == 0) scales[row] = s;
        for (int64_t i = lane; i < nvec; i += 32) {
            float f[PV];
            unpack(src[i], f, T());
            uint32_t w[PV / 4];
            quantize_values<PV>(f, s, rinv, w);
            store_codes<PV>(codes + row * d + i * PV, w);
        }
    }
}

// ---------------------------------------------------------------------------------
// Dequantize.  A warp covers 32 * CPV * K codes; for vector k, lane l owns codes
// [(k*32 + l) * CPV, +CPV), so both the code loads and the output stores of every
// instruction are contiguous across the warp.  CPV = 4 for fp32 output (one 16-byte
// store), 8 for fp16 output (one 16-byte store).  Codes -> fp32 exactly by placing the
// biased byte (c + 128) in the mantissa of 1.5 * 2^23 and subtracting 1.5 * 2^23 + 128.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ float code_to_float(uint32_t biased_word, int byte) {
    const uint32_t u = __byte_perm(biased_word, 0x4B400000u, 0x7650u + byte);
    return __fsub_rn(__uint_as_float(u), kCodeMagic);
}

template <bool F16_OUT>
__global__ void __launch_bounds__(256)
dequantize_kernel(const int8_t* __restrict__ codes, const float* __restrict__ scales,
                  int64_t total, int64_t d, int d_shift, void* __restrict__ out) {
    constexpr int CPV = F16_OUT ? 8 : 4;
    constexpr int K = 4;
    constexpr int64_t PER_WARP = 32 * CPV * K;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp * PER_WARP; base < total; base += n_warps * PER_WARP) {
        uint32_t cw[K][CPV / 4];
        float sc[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t e0 = base + (int64_t)(k * 32 + lane) * CPV;
            if (e0 < total) {
                if constexpr (CPV == 4) {
                    cw[k][0] = __ldcs(reinterpret_cast<const unsigned int*>(codes + e0));
                } else {
                    uint2 t = __ldcs(reinterpret_cast<const uint2*>(codes + e0));
                    cw[k][0] = t.x;
                    cw[k][1] = t.y;
                }
                sc[k] = __ldg(scales + (d_shift >= 0 ? (e0 >> d_shift) : (e0 / d)));
            }
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t e0 = base + (int64_t)(k * 32 + lane) * CPV;
            if (e0 >= total) continue;
            float v[CPV];
#pragma unroll
            for (int w = 0; w < CPV / 4; ++w) {
                const uint32_t b = cw[k][w] ^ 0x80808080u;
#pragma unroll
                for (int e = 0; e < 4; ++e) v[4 * w + e] = __fmul_rn(code_to_float(b, e), sc[k]);
            }
            if constexpr (F16_OUT) {
                __half2 h[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
                __stcs(reinterpret_cast<uint4*>(static_cast<__half*>(out) + e0),
                       *reinterpret_cast<uint4*>(h));
            } else {
                __stcs(reinterpret_cast<float4*>(static_cast<float*>(out) + e0),
                       make_float4(v[0], v[1], v[2], v[3]));
            }
        }
    }
}

// ---------------------------------------------------------------------------------
// INT8 scores: scores_r = sum_j q_j * fl32(c_rj * s_r).  TPR lanes per row, each
// lane takes 16-code chunks (lane + k * TPR); q is staged once per block in shared
// memory as fp32.
// ---------------------------------------------------------------------------------
constexpr int kMaxScoreDim = 8192;

template <int TPR>
__global__ void __launch_bounds__(256)
int8_scores_kernel(const void* __restrict__ q, bool q_f16, const int8_t* __restrict__ codes,
                   const float* __restrict__ scales, int64_t n_rows, int d,
                   float* __restrict__ scores) {
    __shared__ float qs[kMaxScoreDim];
    for (int j = threadIdx.x; j < d; j += blockDim.x)
        qs[j] = q_f16 ? __half2float(static_cast<const __half*>(q)[j])
                      : static_cast<const float*>(q)[j];
    __syncthreads();
    constexpr int GROUPS = 256 / TPR;
    const int lane = threadIdx.x % TPR;
    const int group = threadIdx.x / TPR;
    const int nchunk = d / 16;
    for (int64_t base = (int64_t)blockIdx.x * GROUPS; base < n_rows;
         base += (int64_t)gridDim.x * GROUPS) {
        const int64_t row = base + group;
        float acc = 0.0f;
        if (row < n_rows) {
            const float s = __ldg(scales + row);
            const uint4* src = reinterpret_cast<const uint4*>(codes + row * d);
            for (int c = lane; c < nchunk; c += TPR) {
                const uint4 v = __ldcs(src + c);
                const uint32_t w[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u,
                                       v.z ^ 0x80808080u, v.w ^ 0x80808080u};
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float xh = __fmul_rn(code_to_float(w[i >> 2], i & 3), s);
                    acc = __fmaf_rn(qs[c * 16 + i], xh, acc);
                }
            }
        }
#pragma unroll
        for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (row < n_rows && lane == 0) scores[row] = acc;
    }
}

int grid_for(int64_t work_items, int items_per_block, int blocks_per_sm) {
    const int64_t need = (work_items + items_per_block - 1) / items_per_block;
    const int64_t cap = (int64_t)device_sm_count() * blocks_per_sm;
    int64_t g = need < cap ? need : cap;
    return (int)(g < 1 ? 1 : g);
}

template <typename T, int TPR, int VPT, int RPT>
cudaError_t run_warp(const void* x, int64_t n, int8_t* c, float* s, cudaStream_t st) {
    constexpr int ROWS = (256 / TPR) * RPT;
    quantize_rows_warp<T, TPR, VPT, RPT>
        <<<grid_for(n, ROWS, 8), 256, 0, st>>>(static_cast<const T*>(x), n, c, s);
    return cudaGetLastError();
}

template <typename T, int VPT>
cudaError_t run_cta(const void* x, int64_t n, int8_t* c, float* s, cudaStream_t st) {
    quantize_rows_cta<T, VPT><<<grid_for(n, 1, 8), 256, 0, st>>>(static_cast<const T*>(x), n, c, s);
    return cudaGetLastError();
}

template <typename T>
cudaError_t run_generic(const void* x, int64_t n, int64_t d, int8_t* c, float* s,
                        cudaStream_t st) {
    quantize_rows_generic<T><<<grid_for(n, 8, 8), 256, 0, st>>>(static_cast<const T*>(x), n, d, c, s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_int8(const void* x, bool f16, int64_t n, int64_t d, int8_t* c,
                                 float* s, cudaStream_t st) {
    // Row mappings: each lane holds up to four 16-byte vectors of its row (fewer lanes
    // per row amortise the per-row reduction, scale and reciprocal over more elements).
    if (f16) {
        switch (d) {  // 8 halves per 16-byte vector
            case 16: return run_warp<__half, 2, 1, 4>(x, n, c, s, st);
            case 32: return run_warp<__half, 2, 2, 2>(x, n, c, s, st);
            case 64: return run_warp<__half, 2, 4, 1>(x, n, c, s, st);
            case 128: return run_warp<__half, 4, 4, 1>(x, n, c, s, st);
            case 256: return run_warp<__half, 8, 4, 1>(x, n, c, s, st);
            case 512: return run_warp<__half, 16, 4, 1>(x, n, c, s, st);
            case 1024: return run_warp<__half, 32, 4, 1>(x, n, c, s, st);
            case 2048: return run_cta<__half, 1>(x, n, c, s, st);
            case 4096: return run_cta<__half, 2>(x, n, c, s, st);
            case 8192: return run_cta<__half, 4>(x, n, c, s, st);
            default: return run_generic<__half>(x, n, d, c, s, st);
        }
    }
    switch (d) {  // 4 floats per 16-byte vector
        case 16: return run_warp<float, 2, 2, 2>(x, n, c, s, st);
        case 32: return run_warp<float, 2, 4, 1>(x, n, c, s, st);
        case 64: return run_warp<float, 4, 4, 1>(x, n, c, s, st);
        case 128: return run_warp<float, 8, 4, 1>(x, n, c, s, st);
        case 256: return run_warp<float, 16, 4, 1>(x, n, c, s, st);
        case 512: return run_warp<float, 32, 4, 1>(x, n, c, s, st);
        case 1024: return run_warp<float, 32, 8, 1>(x, n, c, s, st);
        case 2048: return run_cta<float, 2>(x, n, c, s, st);
        case 4096: return run_cta<float, 4>(x, n, c, s, st);
        case 8192: return run_cta<float, 8>(x, n, c, s, st);
        default: return run_generic<float>(x, n, d, c, s, st);
    }
}

cudaError_t launch_dequantize_int8(const int8_t* codes, const float* scales, int64_t n,
                                   int64_t d, void* out, bool f16, cudaStream_t st) {
    const int64_t total = n * d;
    const int per_block = (256 / 32) * 32 * (f16 ? 8 : 4) * 4;
    int shift = -1;
    if ((d & (d - 1)) == 0) {
        shift = 0;
        while ((int64_t(1) << shift) < d) ++shift;
    }
    if (f16)
        dequantize_kernel<true><<<grid_for(total, per_block, 8), 256, 0, st>>>(codes, scales, total, d, shift, out);
    else
        dequantize_kernel<false><<<grid_for(total, per_block, 8), 256, 0, st>>>(codes, scales, total, d, shift, out);
    return cudaGetLastError();
}

cudaError_t launch_int8_scores(const void* q, bool q_f16, const int8_t* codes,
                               const float* scales, int64_t n, int64_t d, float* scores,
                               cudaStream_t st) {
    const int chunks = (int)(d / 16);
    const int di = (int)d;
    if (chunks <= 1) {
        int8_scores_kernel<1><<<grid_for(n, 256, 4), 256, 0, st>>>(q, q_f16, codes, scales, n, di, scores);
    } else if (chunks <= 2) {
        int8_scores_kernel<2><<<grid_for(n, 128, 4), 256, 0, st>>>(q, q_f16, codes, scales, n, di, scores);
    } else if (chunks <= 4) {
        int8_scores_kernel<4><<<grid_for(n, 64, 4), 256, 0, st>>>(q, q_f16, codes, scales, n, di, scores);
    } else if (chunks <= 8) {
        int8_scores_kernel<8><<<grid_for(n, 32, 4), 256, 0, st>>>(q, q_f16, codes, scales, n, di, scores);
    } else if (chunks <= 16) {
        int8_scores_kernel<16><<<grid_for(n, 16, 4), 256, 0, st>>>(q, q_f16, codes, scales, n, di, scores);
    } else {
        int8_scores_kernel<32><<<grid_for(n, 8, 4), 256, 0, st>>>(q, q_f16, codes, scales, n, di, scores);
    }
    return cudaGetLastError();
}

}  // namespace kvq
