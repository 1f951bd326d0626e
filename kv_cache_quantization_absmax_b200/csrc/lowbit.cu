// Channel-wise INT8 and asymmetric group-wise INT4 quantize / dequantize.
//
// Definitions: "Q-TensorFormer" model card, section 6 "Adaptive KV Cache Quantization &
// Attention-Sink Eviction":
//   Symmetric Channel-Wise INT8:  X_hat = clamp(round(X / s8), -128, 127) * s8,
//                                 s8 = max|X| / 127, one s8 per channel (column);
//   Asymmetric Group-Wise INT4:   X_hat = clamp(round((X - z4) / s4), 0, 15) * s4 + z4,
//                                 s4 = (max X - min X) / 15, z4 = min X, per group of
//                                 `group` consecutive elements of a row.
// Codes are bit-identical to the definitions computed in fp32 with IEEE operations and
// round-half-to-even: the quotient takes the reciprocal fast
// path of kvq_int8.cuh and falls back to the IEEE division within 2^-14 of a
// half-integer.  INT4 codes are packed two per byte, element 2i in bits 0-3.
//
// All kernels stream HBM with 16-byte accesses contiguous across each warp.
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_int8.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

// Eight consecutive elements of a row, widened to fp32 (exact from fp16).
template <bool F16>
__device__ __forceinline__ void load8(const void* x, int64_t e0, float* f) {
    if constexpr (F16) {
        const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const __half*>(x) + e0);
        const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __half22float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(x) + e0);
        const uint4 a = p[0], b = p[1];
        f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
        f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
        f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
        f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
    }
}

template <bool F16>
__device__ __forceinline__ void store8(void* out, int64_t e0, const float* f) {
    if constexpr (F16) {
        uint4 v;
        __half2* h = reinterpret_cast<__half2*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        *reinterpret_cast<uint4*>(static_cast<__half*>(out) + e0) = v;
    } else {
        uint4* p = reinterpret_cast<uint4*>(static_cast<float*>(out) + e0);
        p[0] = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
        p[1] = make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]),
                          __float_as_uint(f[7]));
    }
}

// rint_even(fl32(t / s)) clamped to [lo, hi], for one element with its own scale s and
// reciprocal r = scale_reciprocal(s): the fast path when it is provably the same
// integer (see kvq_int8.cuh), else the IEEE division; s == 0 gives 0.
__device__ __forceinline__ int quant1(float t, float s, float r, int lo, int hi) {
    if (s >= i8::kFltMinNormal) {
        const float q = __fmul_rn(t, r);
        const float yf = __fadd_rn(q, i8::kRoundMagic);
        const float d = __fsub_rn(q, __fsub_rn(yf, i8::kRoundMagic));
        if (fabsf(d) <= i8::kTieGuard) {
            // yf = 1.5 * 2^23 + c: its bit pattern is 0x4B400000 + c, whose low 16 bits
            // are c as a 16-bit two's-complement integer
            const int c = (int)(int16_t)(__float_as_uint(yf) & 0xFFFFu);
            return min(max(c, lo), hi);
        }
    } else if (s == 0.0f) {
        return 0;
    }
    const int c = __float2int_rn(__fdiv_rn(t, s));
    return min(max(c, lo), hi);
}

// ---- group-wise INT4: a thread takes 8 elements; LPG = group / 8 lanes per group ----
template <bool F16, int LPG>
__global__ void __launch_bounds__(256) int4_quantize_kernel(const void* __restrict__ x, int64_t n8,
                                                            int group, uint8_t* __restrict__ packed,
                                                            float* __restrict__ scales,
                                                            float* __restrict__ zeros) {
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // every lane of a warp runs the same number of iterations (n8 is a multiple of LPG,
    // and the loop bound is taken per warp) so that the group shuffles stay full
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) - lane;
    for (int64_t base = warp0; base < n8; base += stride) {
        const int64_t i = base + lane;
        const bool live = i < n8;
        float f[8];
        if (live) load8<F16>(x, i * 8, f);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = 0.0f;
        float mn = f[0], mx = f[0];
#pragma unroll
        for (int e = 1; e < 8; ++e) {
            mn = fminf(mn, f[e]);
            mx = fmaxf(mx, f[e]);
        }
#pragma unroll
        for (int off = 1; off < LPG; off <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        if (!live) continue;
        const float s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        const float r = i8::scale_reciprocal(s);
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) word |= (uint32_t)quant1(__fsub_rn(f[e], mn), s, r, 0, 15) << (4 * e);
        *reinterpret_cast<uint32_t*>(packed + i * 4) = word;
        if ((lane & (LPG - 1)) == 0) {
            const int64_t gi = (i * 8) / group;
            scales[gi] = s;
            zeros[gi] = mn;
        }
    }
}

template <bool F16>
__global__ void __launch_bounds__(256) int4_dequantize_kernel(const uint8_t* __restrict__ packed,
                                                              const float* __restrict__ scales,
                                                              const float* __restrict__ zeros, int64_t n8,
                                                              int group, void* __restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const uint32_t word = __ldcs(reinterpret_cast<const unsigned int*>(packed + i * 4));
        const int64_t gi = (i * 8) / group;
        const float s = __ldg(scales + gi), z = __ldg(zeros + gi);
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            f[e] = __fadd_rn(__fmul_rn((float)((word >> (4 * e)) & 0xFu), s), z);
        store8<F16>(out, i * 8, f);
    }
}

// ---- channel-wise INT8: one CTA per (block, 64-column tile); lane l: columns 2l, 2l+1
// of the tile; 8 warps stride over the rows.  Pass 1: column absmax -> scales; pass 2:
// codes. ----
constexpr int kCwCols = 64;
constexpr int kCwWarps = 8;

template <bool F16>
__device__ __forceinline__ float2 load2(const void* x, int64_t i) {
    if constexpr (F16) return __half22float2(*reinterpret_cast<const __half2*>(static_cast<const __half*>(x) + i));
    else return *reinterpret_cast<const float2*>(static_cast<const float*>(x) + i);
}

template <bool F16>
__global__ void __launch_bounds__(32 * kCwWarps) int8_cw_quantize_kernel(const void* __restrict__ x,
                                                                        int64_t rows, int64_t d,
                                                                        int8_t* __restrict__ codes,
                                                                        float* __restrict__ scales) {
    __shared__ float amax[kCwWarps][kCwCols];
    __shared__ float s_sh[kCwCols], r_sh[kCwCols];
    const int64_t blk = blockIdx.y;
    const int64_t c0 = (int64_t)blockIdx.x * kCwCols;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t base = blk * rows * d + c0 + 2 * lane;
    float a0 = 0.0f, a1 = 0.0f;
    for (int64_t r = warp; r < rows; r += kCwWarps) {
        const float2 v = load2<F16>(x, base + r * d);
        a0 = fmaxf(a0, fabsf(v.x));
        a1 = fmaxf(a1, fabsf(v.y));
    }
    amax[warp][2 * lane] = a0;
    amax[warp][2 * lane + 1] = a1;
    __syncthreads();
    if (threadIdx.x < kCwCols) {
        float a = 0.0f;
#pragma unroll
        for (int w = 0; w < kCwWarps; ++w) a = fmaxf(a, amax[w][threadIdx.x]);
        const float s = i8::row_scale(a);
        s_sh[threadIdx.x] = s;
        r_sh[threadIdx.x] = i8::scale_reciprocal(s);
        scales[blk * d + c0 + threadIdx.x] = s;
    }
    __syncthreads();
    const float s0 = s_sh[2 * lane], s1 = s_sh[2 * lane + 1];
    const float r0 = r_sh[2 * lane], r1 = r_sh[2 * lane + 1];
    for (int64_t r = warp; r < rows; r += kCwWarps) {
        const float2 v = load2<F16>(x, base + r * d);
        const uint32_t c = (uint32_t)(quant1(v.x, s0, r0, -128, 127) & 0xFF) |
                           ((uint32_t)(quant1(v.y, s1, r1, -128, 127) & 0xFF) << 8);
        *reinterpret_cast<uint16_t*>(codes + base + r * d) = (uint16_t)c;
    }
}

template <bool F16>
__global__ void __launch_bounds__(256) int8_cw_dequantize_kernel(const int8_t* __restrict__ codes,
                                                                 const float* __restrict__ scales,
                                                                 int64_t rows, int64_t d, int64_t n16,
                                                                 void* __restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
        const int64_t e0 = i * 16;
        const uint4 cv = __ldcs(reinterpret_cast<const uint4*>(codes + e0));
        const int8_t* c = reinterpret_cast<const int8_t*>(&cv);
        const int64_t blk = e0 / (rows * d);
        const int64_t col = e0 % d;
        const float* sc = scales + blk * d + col;
        float f[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = __fmul_rn((float)c[e], __ldg(sc + e));
        store8<F16>(out, e0, f);
        store8<F16>(out, e0 + 8, f + 8);
    }
}

unsigned grid_for(int64_t items, int threads) {
    const int64_t want = (items + threads - 1) / threads;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    return (unsigned)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_quantize_int4(const void* x, bool f16, int64_t n_rows, int64_t d, int group,
                                 uint8_t* packed, float* scales, float* zeros, cudaStream_t st) {
    const int64_t n8 = n_rows * d / 8;
    if (n8 == 0) return cudaSuccess;
    const unsigned grid = grid_for(n8, 256);
    switch (group * 2 + (f16 ? 1 : 0)) {
        case 64: int4_quantize_kernel<false, 4><<<grid, 256, 0, st>>>(x, n8, group, packed, scales, zeros); break;
        case 65: int4_quantize_kernel<true, 4><<<grid, 256, 0, st>>>(x, n8, group, packed, scales, zeros); break;
        case 128: int4_quantize_kernel<false, 8><<<grid, 256, 0, st>>>(x, n8, group, packed, scales, zeros); break;
        case 129: int4_quantize_kernel<true, 8><<<grid, 256, 0, st>>>(x, n8, group, packed, scales, zeros); break;
        case 256: int4_quantize_kernel<false, 16><<<grid, 256, 0, st>>>(x, n8, group, packed, scales, zeros); break;
        case 257: int4_quantize_kernel<true, 16><<<grid, 256, 0, st>>>(x, n8, group, packed, scales, zeros); break;
        default: return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize_int4(const uint8_t* packed, const float* scales, const float* zeros,
                                   int64_t n_rows, int64_t d, int group, void* out, bool f16,
                                   cudaStream_t st) {
    const int64_t n8 = n_rows * d / 8;
    if (n8 == 0) return cudaSuccess;
    const unsigned grid = grid_for(n8, 256);
    if (f16) int4_dequantize_kernel<true><<<grid, 256, 0, st>>>(packed, scales, zeros, n8, group, out);
    else int4_dequantize_kernel<false><<<grid, 256, 0, st>>>(packed, scales, zeros, n8, group, out);
    return cudaGetLastError();
}

cudaError_t launch_quantize_int8_channelwise(const void* x, bool f16, int64_t n_blocks, int64_t rows,
                                             int64_t d, int8_t* codes, float* scales, cudaStream_t st) {
    if (n_blocks == 0) return cudaSuccess;
    const dim3 grid((unsigned)(d / kCwCols), (unsigned)n_blocks);
    if (f16) int8_cw_quantize_kernel<true><<<grid, 32 * kCwWarps, 0, st>>>(x, rows, d, codes, scales);
    else int8_cw_quantize_kernel<false><<<grid, 32 * kCwWarps, 0, st>>>(x, rows, d, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_dequantize_int8_channelwise(const int8_t* codes, const float* scales, int64_t n_blocks,
                                               int64_t rows, int64_t d, void* out, bool f16,
                                               cudaStream_t st) {
    const int64_t n16 = n_blocks * rows * d / 16;
    if (n16 == 0) return cudaSuccess;
    const unsigned grid = grid_for(n16, 256);
    if (f16) int8_cw_dequantize_kernel<true><<<grid, 256, 0, st>>>(codes, scales, rows, d, n16, out);
    else int8_cw_dequantize_kernel<false><<<grid, 256, 0, st>>>(codes, scales, rows, d, n16, out);
    return cudaGetLastError();
}

}  // namespace kvq
