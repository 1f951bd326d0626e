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

#include "kvq_f32x2.cuh"
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

// (streaming stores: the outputs are not read again by the kernel)
template <bool F16>
__device__ __forceinline__ void store8(void* out, int64_t e0, const float* f) {
    if constexpr (F16) {
        uint4 v;
        __half2* h = reinterpret_cast<__half2*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        __stcs(reinterpret_cast<uint4*>(static_cast<__half*>(out) + e0), v);
    } else {
        uint4* p = reinterpret_cast<uint4*>(static_cast<float*>(out) + e0);
        __stcs(p, make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                             __float_as_uint(f[3])));
        __stcs(p + 1, make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]),
                                 __float_as_uint(f[7])));
    }
}

// Quantizing 8 values t_e with scales s_e (reciprocals r_e = scale_reciprocal(s_e)):
// code = rint_even(fl32(t_e / s_e)) clamped to the range.  The reciprocal fast path
// serves all 8 when every scale is normal and every quotient is provably rounded the
// same way (kvq_int8.cuh); its codes need no clamp (|t / s| <= 127 (1 + 2^-23) for
// INT8, 0 <= t / s <= 15 (1 + 2^-23) for INT4) and are the low bits of the sums
// y_e = 1.5 * 2^23 + code.  Otherwise each value takes the IEEE division (a zero scale
// gives 0).  Branch-free on the fast path.
// The fast path runs on fp32x2 pairs: q = t r, y = q + M, and the rounding error
// q - (y - M) computed as q + (M - y), where M - y = fma(y, -1, M) is exact (y and M
// are within a factor of two), so every value is the scalar sequence's.
template <bool UNIFORM>
__device__ __forceinline__ bool fast_sums(const float* t, const float* sc, const float* rc, uint32_t* y) {
    using namespace x2;
    const uint64_t magic2 = pack2(i8::kRoundMagic, i8::kRoundMagic);
    const uint64_t mone2 = pack2(-1.0f, -1.0f);
    float tmax = 0.0f;
    float smin = sc[0];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        const uint64_t r2 = UNIFORM ? pack2(rc[0], rc[0]) : pack2(rc[e], rc[e + 1]);
        const uint64_t q2 = mul2(pack2(t[e], t[e + 1]), r2);
        const uint64_t y2 = add2(q2, magic2);
        const float2 d = unpack2(add2(q2, fma2(y2, mone2, magic2)));
        tmax = fmaxf(tmax, fmaxf(fabsf(d.x), fabsf(d.y)));
        const float2 yy = unpack2(y2);
        y[e] = __float_as_uint(yy.x);
        y[e + 1] = __float_as_uint(yy.y);
        if (!UNIFORM) smin = fminf(smin, fminf(sc[e], sc[e + 1]));
    }
    return smin >= i8::kFltMinNormal && tmax <= i8::kTieGuard;
}

// INT8 codes of 8 values with their own scales -> 8 bytes.
__device__ __forceinline__ uint2 quant8_i8(const float* t, const float* sc, const float* rc) {
    uint32_t y[8];
    if (!fast_sums<false>(t, sc, rc, y)) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            y[e] = sc[e] == 0.0f ? 0u : (uint32_t)min(max(__float2int_rn(__fdiv_rn(t[e], sc[e])), -128), 127);
    }
    return make_uint2(i8::pack_low_bytes(y[0], y[1], y[2], y[3]), i8::pack_low_bytes(y[4], y[5], y[6], y[7]));
}

// INT4 codes of 8 values sharing scale s -> one word, value e in bits 4e .. 4e + 3.
__device__ __forceinline__ uint32_t quant8_u4(const float* t, float s, float r) {
    uint32_t y[8];
    if (!fast_sums<true>(t, &s, &r, y)) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            y[e] = s == 0.0f ? 0u : (uint32_t)min(max(__float2int_rn(__fdiv_rn(t[e], s)), 0), 15);
    }
    // bytes [c0, c1, c2, c3] -> x = b | (b >> 4) has c0 | c1 << 4 in byte 0 and
    // c2 | c3 << 4 in byte 2 (every code < 16)
    const uint32_t b03 = i8::pack_low_bytes(y[0], y[1], y[2], y[3]);
    const uint32_t b47 = i8::pack_low_bytes(y[4], y[5], y[6], y[7]);
    return __byte_perm(b03 | (b03 >> 4), b47 | (b47 >> 4), 0x6420);
}

// ---- group-wise INT4: a lane takes 32 consecutive elements (one group of 32, half a
// group of 64, a quarter of a group of 128: LPG = group / 32 lanes per group). ----
template <bool F16>
__device__ __forceinline__ void load32(const void* x, int64_t e0, float* f, float& mn, float& mx) {
    if constexpr (F16) {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __half*>(x) + e0);
        uint4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = p[k];
        const __half2* h = reinterpret_cast<const __half2*>(v);
        __half2 lo = h[0], hi = h[0];
#pragma unroll
        for (int k = 1; k < 16; ++k) {
            lo = __hmin2(lo, h[k]);
            hi = __hmax2(hi, h[k]);
        }
        mn = fminf(__low2float(lo), __high2float(lo));
        mx = fmaxf(__low2float(hi), __high2float(hi));
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float2 t = __half22float2(h[k]);
            f[2 * k] = t.x;
            f[2 * k + 1] = t.y;
        }
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(x) + e0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint4 v = p[k];
            f[4 * k] = __uint_as_float(v.x);
            f[4 * k + 1] = __uint_as_float(v.y);
            f[4 * k + 2] = __uint_as_float(v.z);
            f[4 * k + 3] = __uint_as_float(v.w);
        }
        mn = f[0];
        mx = f[0];
#pragma unroll
        for (int e = 1; e < 32; ++e) {
            mn = fminf(mn, f[e]);
            mx = fmaxf(mx, f[e]);
        }
    }
}

// RES: also write the residual of each element against its INT4 reconstruction,
// fp16(fl32(x - fl32(fl32(c * s) + z))), to resid (same layout as x; fp16 x only).
template <bool F16, int LPG, bool RES = false>
__global__ void __launch_bounds__(256) int4_quantize_kernel(const void* __restrict__ x, int64_t n32,
                                                            uint8_t* __restrict__ packed,
                                                            float* __restrict__ scales,
                                                            float* __restrict__ zeros,
                                                            __half* __restrict__ resid = nullptr) {
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // the loop bound is warp-uniform (n32 is a multiple of LPG and every warp starts on a
    // multiple of 32), so the group shuffles always see full warps
    for (int64_t base = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) - lane; base < n32; base += stride) {
        const int64_t i = base + lane;
        const bool live = i < n32;
        float f[32];
        float mn = 0.0f, mx = 0.0f;
        if (live) load32<F16>(x, i * 32, f, mn, mx);
#pragma unroll
        for (int off = 1; off < LPG; off <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        if (!live) continue;
        const float s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        const float r = i8::scale_reciprocal(s);
        const uint64_t nmn2 = x2::pack2(-mn, -mn);
        uint32_t word[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float t[8];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {   // t = fl32(x - z4), pairwise
                const float2 tt = x2::unpack2(x2::add2(x2::pack2(f[8 * c + e], f[8 * c + e + 1]), nmn2));
                t[e] = tt.x;
                t[e + 1] = tt.y;
            }
            word[c] = quant8_u4(t, s, r);
        }
        *reinterpret_cast<uint4*>(packed + i * 16) = make_uint4(word[0], word[1], word[2], word[3]);
        if constexpr (RES) {
            // k_hat = fl32(fl32(c * s) + z), r = fp16(fl32(x - k_hat)): scalar IEEE
            // operations, each rounded on its own (never contracted into an fma)
            uint4 out[4];
            uint32_t* o = reinterpret_cast<uint32_t*>(out);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const uint32_t w = word[e >> 3];
                const float c0 = (float)((w >> (4 * (e & 7))) & 0xFu);
                const float c1 = (float)((w >> (4 * ((e & 7) + 1))) & 0xFu);
                const float r0 = __fsub_rn(f[e], __fadd_rn(__fmul_rn(c0, s), mn));
                const float r1 = __fsub_rn(f[e + 1], __fadd_rn(__fmul_rn(c1, s), mn));
                const __half2 h = __floats2half2_rn(r0, r1);
                o[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            }
            uint4* dst = reinterpret_cast<uint4*>(resid + i * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = out[k];
        }
        if ((lane & (LPG - 1)) == 0) {
            const int64_t gi = i / LPG;   // group index: 32 LPG elements per group
            scales[gi] = s;
            zeros[gi] = mn;
        }
    }
}

// INT4 dequantize: a lane takes chunks of 8 elements (one packed word, one 16-byte
// fp16 store), lane-contiguous, 4 chunks per lane in flight; g8_shift = log2(group / 8).
template <bool F16>
__global__ void __launch_bounds__(256) int4_dequantize_kernel(const uint8_t* __restrict__ packed,
                                                              const float* __restrict__ scales,
                                                              const float* __restrict__ zeros, int64_t n8,
                                                              int g8_shift, void* __restrict__ out) {
    constexpr int K = 4;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp * 32 * K; base < n8; base += n_warps * 32 * K) {
        uint32_t w[K];
        float sc[K], zc[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t i = base + 32 * k + lane;
            if (i < n8) {
                w[k] = __ldcs(reinterpret_cast<const unsigned int*>(packed) + i);
                sc[k] = __ldg(scales + (i >> g8_shift));
                zc[k] = __ldg(zeros + (i >> g8_shift));
            }
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t i = base + 32 * k + lane;
            if (i >= n8) continue;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __fadd_rn(__fmul_rn((float)((w[k] >> (4 * e)) & 0xFu), sc[k]), zc[k]);
            store8<F16>(out, i * 8, f);
        }
    }
}

// ---- channel-wise INT8: persistent CTAs of 512 threads (one per SM) walk the
// (block, 64-column tile) items.  Thread (row group rg = tid / 8, column chunk
// cg = tid % 8) takes columns 8 cg .. 8 cg + 7 of rows rg, rg + 64, ...  Pass 1: column
// absmax -> scales; pass 2: codes.  A CTA's tile (rows x 128 B for fp16) is re-read
// right after it was read, and with one tile per SM in flight (76 MB for 4096-row fp16
// tiles) the second pass reads L2. ----
constexpr int kCwCols = 64;
constexpr int kCwThreads = 512;
constexpr int kCwRowGroups = kCwThreads / 8;
constexpr int kCwP1 = 4;
constexpr int kCwP2 = 2;

template <bool F16>
__global__ void __launch_bounds__(kCwThreads, 1) int8_cw_quantize_kernel(const void* __restrict__ x,
                                                                        int64_t n_blocks, int64_t rows,
                                                                        int64_t d, int8_t* __restrict__ codes,
                                                                        float* __restrict__ scales) {
    __shared__ float amax[kCwRowGroups][kCwCols + 1];
    __shared__ float s_sh[kCwCols], r_sh[kCwCols];
    const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
    const int64_t tiles = d / kCwCols;
    for (int64_t item = blockIdx.x; item < n_blocks * tiles; item += gridDim.x) {
        const int64_t blk = item / tiles;
        const int64_t c0 = (item % tiles) * kCwCols;
        const int64_t base = blk * rows * d + c0 + 8 * cg;
        float a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = 0.0f;
        // kCwP1 rows per thread in flight in the column-max pass, kCwP2 in the code pass
        for (int64_t r = rg; r < rows; r += kCwP1 * kCwRowGroups) {
            float f[kCwP1][8];
#pragma unroll
            for (int k = 0; k < kCwP1; ++k) {
                if (r + k * kCwRowGroups < rows) load8<F16>(x, base + (r + k * kCwRowGroups) * d, f[k]);
                else
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[k][e] = 0.0f;
            }
#pragma unroll
            for (int k = 0; k < kCwP1; ++k)
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = fmaxf(a[e], fabsf(f[k][e]));
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) amax[rg][8 * cg + e] = a[e];
        __syncthreads();
        if (threadIdx.x < kCwCols) {
            float m = 0.0f;
            for (int g = 0; g < kCwRowGroups; ++g) m = fmaxf(m, amax[g][threadIdx.x]);
            const float s = i8::row_scale(m);
            s_sh[threadIdx.x] = s;
            r_sh[threadIdx.x] = i8::scale_reciprocal(s);
            scales[blk * d + c0 + threadIdx.x] = s;
        }
        __syncthreads();
        float sc[8], rc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sc[e] = s_sh[8 * cg + e];
            rc[e] = r_sh[8 * cg + e];
        }
        for (int64_t r = rg; r < rows; r += kCwP2 * kCwRowGroups) {
            float f[kCwP2][8];
#pragma unroll
            for (int k = 0; k < kCwP2; ++k)
                if (r + k * kCwRowGroups < rows) load8<F16>(x, base + (r + k * kCwRowGroups) * d, f[k]);
#pragma unroll
            for (int k = 0; k < kCwP2; ++k) {
                if (r + k * kCwRowGroups >= rows) continue;
                *reinterpret_cast<uint2*>(codes + base + (r + k * kCwRowGroups) * d) = quant8_i8(f[k], sc, rc);
            }
        }
        __syncthreads();  // amax / s_sh are rewritten by the next item
    }
}

// channel-wise dequantize: grid.y = block; a lane takes chunks of 8 consecutive codes
// (lane-contiguous 8-byte loads and 16-byte fp16 stores, 4 chunks in flight) and their
// 8 column scales (two 16-byte loads, cached).
template <bool F16>
__global__ void __launch_bounds__(256) int8_cw_dequantize_kernel(const int8_t* __restrict__ codes,
                                                                 const float* __restrict__ scales,
                                                                 int64_t rows, int64_t d,
                                                                 void* __restrict__ out) {
    constexpr int K = 4;
    const int64_t blk = blockIdx.y;
    const uint32_t n8 = (uint32_t)(rows * d / 8);        // chunks of one block (< 2^32)
    const uint32_t d8 = (uint32_t)(d / 8);                // chunks per row
    const int8_t* cb = codes + blk * rows * d;
    const float* sb = scales + blk * d;
    const int64_t ob = blk * rows * d;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t base = warp * 32 * K; base < n8; base += n_warps * 32 * K) {
        uint2 cv[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const uint32_t i = base + 32 * k + lane;
            if (i < n8) cv[k] = __ldcs(reinterpret_cast<const uint2*>(cb) + i);
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const uint32_t i = base + 32 * k + lane;
            if (i >= n8) continue;
            const float4* sc = reinterpret_cast<const float4*>(sb + (i % d8) * 8u);  // column of chunk i
            const float4 s0 = __ldg(sc), s1 = __ldg(sc + 1);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            const int8_t* c = reinterpret_cast<const int8_t*>(&cv[k]);
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __fmul_rn((float)c[e], sv[e]);
            store8<F16>(out, ob + (int64_t)i * 8, f);
        }
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
    const int64_t n32 = n_rows * d / 32;
    if (n32 == 0) return cudaSuccess;
    const unsigned grid = grid_for(n32, 256);
    switch (group * 2 + (f16 ? 1 : 0)) {
        case 64: int4_quantize_kernel<false, 1><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros); break;
        case 65: int4_quantize_kernel<true, 1><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros); break;
        case 128: int4_quantize_kernel<false, 2><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros); break;
        case 129: int4_quantize_kernel<true, 2><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros); break;
        case 256: int4_quantize_kernel<false, 4><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros); break;
        case 257: int4_quantize_kernel<true, 4><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros); break;
        default: return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_int4_residual(const uint16_t* x, int64_t n_rows, int64_t d, int group,
                                          uint8_t* packed, float* scales, float* zeros, uint16_t* resid,
                                          cudaStream_t st) {
    const int64_t n32 = n_rows * d / 32;
    if (n32 == 0) return cudaSuccess;
    const unsigned grid = grid_for(n32, 256);
    __half* r = reinterpret_cast<__half*>(resid);
    switch (group) {
        case 32: int4_quantize_kernel<true, 1, true><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros, r); break;
        case 64: int4_quantize_kernel<true, 2, true><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros, r); break;
        case 128: int4_quantize_kernel<true, 4, true><<<grid, 256, 0, st>>>(x, n32, packed, scales, zeros, r); break;
        default: return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize_int4(const uint8_t* packed, const float* scales, const float* zeros,
                                   int64_t n_rows, int64_t d, int group, void* out, bool f16,
                                   cudaStream_t st) {
    const int64_t n8 = n_rows * d / 8;
    if (n8 == 0) return cudaSuccess;
    const unsigned grid = grid_for((n8 + 3) / 4, 256);
    const int g8_shift = group == 32 ? 2 : (group == 64 ? 3 : 4);
    if (f16) int4_dequantize_kernel<true><<<grid, 256, 0, st>>>(packed, scales, zeros, n8, g8_shift, out);
    else int4_dequantize_kernel<false><<<grid, 256, 0, st>>>(packed, scales, zeros, n8, g8_shift, out);
    return cudaGetLastError();
}

cudaError_t launch_quantize_int8_channelwise(const void* x, bool f16, int64_t n_blocks, int64_t rows,
                                             int64_t d, int8_t* codes, float* scales, cudaStream_t st) {
    const int64_t items = n_blocks * (d / kCwCols);
    if (items == 0) return cudaSuccess;
    const int64_t sms = device_sm_count();
    const unsigned grid = (unsigned)(items < sms ? items : sms);
    if (f16) int8_cw_quantize_kernel<true><<<grid, kCwThreads, 0, st>>>(x, n_blocks, rows, d, codes, scales);
    else int8_cw_quantize_kernel<false><<<grid, kCwThreads, 0, st>>>(x, n_blocks, rows, d, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_dequantize_int8_channelwise(const int8_t* codes, const float* scales, int64_t n_blocks,
                                               int64_t rows, int64_t d, void* out, bool f16,
                                               cudaStream_t st) {
    if (n_blocks == 0) return cudaSuccess;
    const int64_t n8 = rows * d / 8;
    const int64_t want = (n8 + 1023) / 1024;               // 256 threads x 4 chunks
    const int64_t per_block_cap = n_blocks >= 1184 ? 1 : (1184 + n_blocks - 1) / n_blocks;
    const dim3 grid((unsigned)(want < per_block_cap ? want : per_block_cap), (unsigned)n_blocks);
    if (f16) int8_cw_dequantize_kernel<true><<<grid, 256, 0, st>>>(codes, scales, rows, d, out);
    else int8_cw_dequantize_kernel<false><<<grid, 256, 0, st>>>(codes, scales, rows, d, out);
    return cudaGetLastError();
}

}  // namespace kvq
