// QJL key sketch and query sketch on the 5th-generation tensor cores (tcgen05).
//
// Definition: "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with Zero
// Overhead", abstract -- the key is projected by a Gaussian JL matrix S and only the
// signs of the projection are kept (sign-bit quantization); the query is projected by
// the same S without quantization; the key's norm is kept for the estimator.
//
// u = K S^T for a tile of 128 keys is one dense [128 x 128] x [128 x m] contraction,
// so it runs as tcgen05.mma (kind::f16, fp16 x fp16 -> fp32 accumulators in tensor
// memory).  Persistent kernel, one CTA per SM, three warp roles:
//   warp 0      TMA producer: S once (it stays in shared memory), then 128-key tiles
//               into a 5-stage ring (two 64-column boxes per tile, 128-byte swizzle);
//   warp 1      allocates 512 TMEM columns (two m-column accumulators), one thread
//               issues 8 MMAs (K = 16 each) per tile and commits to an mbarrier;
//   warps 2..9  two epilogue warpgroups; warpgroup e takes the tiles i with i % 2 == e
//               and always the accumulator e: tcgen05.ld of the accumulator row (one
//               key per thread), sign bits -> packed words (four independent
//               funnel-shift chains per word), the key norm from the tile still in
//               shared memory, 16-byte stores.
// The epilogue computes the tile's norms from shared memory as soon as the tile has
// landed (while the MMA runs), returns the stage to the producer as soon as the MMA is
// done, then packs the sign bits.  The epilogue of tile i overlaps the MMA of tile i+1
// (double-buffered accumulator) and the TMA loads of tiles i+1..i+5 (five stages); each
// warpgroup has two tiles' time for one.
//
// Norms: the stored norm is the fp16 rounding of the fp64 norm whose sum of squares
// is accumulated in index order.  The fast path sums the exact fp32 squares (fp16
// squares fit in fp32) in a fixed tree (at most 11 roundings on any term's path, so
// relative error <= gamma_11 ~ 11 u, u = 2^-24), takes the IEEE root (root of the sum's
// error 5.5 u, plus u for the root's rounding) and checks that n (1 - 2^-21) and
// n (1 + 2^-21) round to the same fp16 value (8 u covers those 6.5 u, the u of the
// product's rounding and the fp64 reference's 2^-46); then that value is the rounding
// of the fp64 norm.  Otherwise (about one key in 600 of LogNormal keys) the key is
// queued in shared memory and, once the CTA's tiles are done, the epilogue threads
// redo those sums in fp64 in index order, one key per thread, reading the keys from
// global memory: a dependent chain of 128 fp64 operations costs about a microsecond,
// and run inline it would hold its whole warp (and through it the accumulator and the
// stage) while 31 lanes idle.  A key that finds the queue full takes the same sum
// inline from the tile in shared memory.
// Sign bits: bit = 1 iff the fp32 accumulator's sign bit is clear.  An exactly zero
// projection of a nonzero key lies inside the tolerance band whatever its sign; a zero
// key (sum of squares 0) gets all bits set, since every projection is exactly 0.
//
// Every mbarrier wait is bounded: after 2 s of global time the waiting role records an
// error code in g_kvq_device_error, raises a CTA-wide abort flag and leaves its loop;
// the producer then waits (bounded) for its own TMA loads still in flight, the MMA
// thread for its own MMAs, and TMEM is freed before the CTA exits.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

__device__ unsigned int g_kvq_device_error = 0;

namespace {

constexpr int kBM = 128;                 // keys per tile (MMA M)
constexpr int kDim = 128;                // head_dim (MMA K in total)
constexpr int kStages = 5;
constexpr int kHalfBytes = kBM * 64 * 2; // one 64-column box of a key tile: 16 KB
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr int kThreads = 320;             // producer, MMA, 2 x 4 epilogue warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;     // TMEM columns between the two accumulators
constexpr int kSlowCap = 256;            // keys whose norm is deferred to the slow path, per CTA

enum : unsigned int {
    kErrProducer = 0x101,
    kErrMma = 0x102,
    kErrEpilogue = 0x103,
    kErrDrain = 0x104,
};

// --------------------------------------------------------------------------------
// PTX wrappers
// --------------------------------------------------------------------------------
using dev::mbar_arrive;
using dev::mbar_arrive_expect_tx;
using dev::mbar_drain;
using dev::mbar_init;
using dev::mbar_try_wait;
using dev::smem_u32;

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int err) {
    return dev::mbar_wait(bar, parity, abort_flag, &g_kvq_device_error, err);
}

using dev::smem_desc_sw128;
using dev::tc_commit;
using dev::tc_fence_after;
using dev::tc_fence_before;
using dev::tc_mma_f16;
using dev::tma_load_2d;
using dev::tmem_alloc;
using dev::tmem_dealloc;
using dev::tmem_ld_32x32b_x32;
using dev::tmem_ld_wait;

// Instruction descriptor, kind::f16: fp32 accumulate, fp16 A and B, both K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

// Bit i of the result = 1 iff r[i] (an fp32 bit pattern) has its sign bit clear.
// Four independent chains of eight funnel shifts keep the dependency chain short.
__device__ __forceinline__ uint32_t pack_nonneg_bits(const uint32_t* r) {
    uint32_t n0 = 0, n1 = 0, n2 = 0, n3 = 0;
#pragma unroll
    for (int j = 7; j >= 0; --j) {
        n0 = __funnelshift_l(r[j], n0, 1);
        n1 = __funnelshift_l(r[8 + j], n1, 1);
        n2 = __funnelshift_l(r[16 + j], n2, 1);
        n3 = __funnelshift_l(r[24 + j], n3, 1);
    }
    return ~(n0 | (n1 << 8) | (n2 << 16) | (n3 << 24));
}

// 16-byte chunk c (of 16) of key row `row` in a swizzled [128 x 128] fp16 tile.
__device__ __forceinline__ uint4 tile_chunk(const uint8_t* st, int row, int c) {
    const int kb = c >> 3, cc = c & 7;
    return *reinterpret_cast<const uint4*>(st + kb * kHalfBytes + row * 128 + ((cc ^ (row & 7)) << 4));
}

// acc + h * h with an fp16 h: the product is exact in fp32 (11-bit significands) and the
// sum is rounded once (mixed-precision FMA, no conversion instruction).
__device__ __forceinline__ float fma_sq_f16(uint16_t h, float acc) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %1, %2;" : "=f"(d) : "h"(h), "f"(acc));
    return d;
}

// Sum of the 128 squares of a key row in fp32: each square is exact; 16 chunk sums of
// 8 terms (8 sequential FMAs), then a 4-level tree: relative error <= 12 u.
__device__ __forceinline__ float row_sum_squares(const uint8_t* st, int row) {
    float s[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint4 v = tile_chunk(st, row, c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a = fma_sq_f16((uint16_t)(w[i] & 0xFFFFu), a);
            a = fma_sq_f16((uint16_t)(w[i] >> 16), a);
        }
        s[c] = a;
    }
#pragma unroll
    for (int step = 8; step >= 1; step >>= 1)
#pragma unroll
        for (int i = 0; i < step; ++i) s[i] = __fadd_rn(s[i], s[i + step]);
    return s[0];
}

// The fp32 fast path: true, with the fp16 bits of the norm, when both ends of
// n (1 -+ 2^-21) round to the same fp16 value.
__device__ __forceinline__ bool norm_f16_fast(float ss, uint16_t& bits) {
    const float n = __fsqrt_rn(ss);
    const __half lo = __float2half_rn(__fmul_rn(n, 1.0f - 0x1p-21f));
    const __half hi = __float2half_rn(__fmul_rn(n, 1.0f + 0x1p-21f));
    bits = __half_as_ushort(lo);
    return __half_as_ushort(lo) == __half_as_ushort(hi);
}

// The defining sequence: fp64 sum of the squares in index order, IEEE root, one
// rounding to fp16.  chunk(c) gives the c-th 8 components (16 bytes) of the key.
template <class Chunk>
__device__ __forceinline__ uint16_t norm_f16_index_order(Chunk chunk) {
    double s64 = 0.0;
#pragma unroll 1
    for (int c = 0; c < 16; ++c) {
        const uint4 x = chunk(c);
        const __half* h = reinterpret_cast<const __half*>(&x);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double d = (double)__half2float(h[i]);
            s64 = __fma_rn(d, d, s64);
        }
    }
    return __half_as_ushort(__double2half(__dsqrt_rn(s64)));
}

struct Smem {
    uint32_t s_base;      // S: two 64-column halves of m rows x 128 B
    uint32_t stage_base;  // key stages
    uint32_t bars;        // mbarriers
};

template <bool kSketchOut>
__global__ void __launch_bounds__(kThreads, 1)
qjl_mma_kernel(const __grid_constant__ CUtensorMap tmap_rows,
               const __grid_constant__ CUtensorMap tmap_s, const uint16_t* __restrict__ rows,
               int64_t n_rows, int m, uint32_t* __restrict__ words,
               uint16_t* __restrict__ norms, float* __restrict__ sketch_out) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag_storage;
    __shared__ int slow_count;
    __shared__ uint32_t slow_keys[kSlowCap];
    volatile int* abort_flag = &abort_flag_storage;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* base_ptr = smem_raw + (base - raw);
    const uint32_t s_half_bytes = (uint32_t)m * 128u;
    const uint32_t s_base = base;
    const uint32_t stage_base = base + 2u * s_half_bytes;
    const uint32_t bar_base = stage_base + kStages * kTileBytes;
    auto full_bar = [&](int s) { return bar_base + 8u * s; };
    auto empty_bar = [&](int s) { return bar_base + 8u * (kStages + s); };
    auto tfull_bar = [&](int a) { return bar_base + 8u * (2 * kStages + a); };
    auto tempty_bar = [&](int a) { return bar_base + 8u * (2 * kStages + 2 + a); };
    const uint32_t s_bar = bar_base + 8u * (2 * kStages + 4);
    const uint32_t done_bar = bar_base + 8u * (2 * kStages + 5);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t n_tiles = (n_rows + kBM - 1) / kBM;

    if (threadIdx.x == 0) {
        abort_flag_storage = 0;
        slow_count = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 4);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 4);
        }
        mbar_init(s_bar, 1);
        mbar_init(done_bar, 1);
        dev::mbar_init_fence();
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_rows)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_s)) : "memory");
            mbar_arrive_expect_tx(s_bar, 2u * s_half_bytes);
            tma_load_2d(s_base, &tmap_s, s_bar, 0, 0);
            tma_load_2d(s_base + s_half_bytes, &tmap_s, s_bar, 64, 0);
            uint32_t issued_parity[kStages];
            bool issued[kStages];
            for (int s = 0; s < kStages; ++s) issued[s] = false, issued_parity[s] = 0;
            int it = 0;
            for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
                const int stage = it % kStages;
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                if (!mbar_wait(empty_bar(stage), ph ^ 1u, abort_flag, kErrProducer)) break;
                const uint32_t dst = stage_base + (uint32_t)stage * kTileBytes;
                mbar_arrive_expect_tx(full_bar(stage), (uint32_t)kTileBytes);
                tma_load_2d(dst, &tmap_rows, full_bar(stage), 0, (int)(tile * kBM));
                tma_load_2d(dst + kHalfBytes, &tmap_rows, full_bar(stage), 64, (int)(tile * kBM));
                issued[stage] = true;
                issued_parity[stage] = ph;
            }
            // Never leave the CTA with a TMA write in flight.
            mbar_drain(s_bar, 0);
            for (int s = 0; s < kStages; ++s)
                if (issued[s]) mbar_drain(full_bar(s), issued_parity[s]);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(m);
            bool ok = mbar_wait(s_bar, 0, abort_flag, kErrMma);
            int it = 0;
            for (int64_t tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++it) {
                const int stage = it % kStages;
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                const int acc = it & 1;
                const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                if (!mbar_wait(full_bar(stage), ph, abort_flag, kErrMma)) break;
                if (!mbar_wait(tempty_bar(acc), aph ^ 1u, abort_flag, kErrMma)) break;
                tc_fence_after();
                const uint32_t a0 = stage_base + (uint32_t)stage * kTileBytes;
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * kAccStride;
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t ad = smem_desc_sw128(a0 + kb * kHalfBytes + k * 32);
                        const uint64_t bd = smem_desc_sw128(s_base + kb * s_half_bytes + k * 32);
                        tc_mma_f16(d_tmem, ad, bd, idesc, (kb | k) != 0);
                    }
                }
                tc_commit(tfull_bar(acc));
            }
            // Wait for every MMA this thread issued before TMEM can be released.
            tc_commit(done_bar);
            mbar_drain(done_bar, 0);
        }
    } else {
        // ---------------- epilogue (warps 2..9) ----------------
        const int eg = (warp - 2) >> 2;          // warpgroup: handles tiles it % 2 == eg
        const int quarter = warp & 3;            // TMEM lanes this warp may access
        const int row = quarter * 32 + lane;     // key row within the tile
        const int nw = m / 32;
        int it = 0;
        for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
            if ((it & 1) != eg) continue;
            const int stage = it % kStages;
            const int acc = eg;
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            const int64_t key = tile * kBM + row;
            float ss = 0.0f;
            uint16_t nbits = 0;
            bool deferred = false;
            if constexpr (!kSketchOut) {
                // The norm needs only the landed tile: compute it while the MMA runs.
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                const bool okf = mbar_wait(full_bar(stage), ph, abort_flag, kErrEpilogue);
                if (!__all_sync(0xffffffffu, okf)) break;
                const uint8_t* st = base_ptr + (stage_base - base) + (size_t)stage * kTileBytes;
                ss = row_sum_squares(st, row);
                if (!norm_f16_fast(ss, nbits) && key < n_rows) {
                    const int slot = key <= 0xFFFFFFFFll ? atomicAdd(&slow_count, 1) : kSlowCap;
                    if (slot < kSlowCap) {
                        slow_keys[slot] = (uint32_t)key;
                        deferred = true;
                    } else {
                        nbits = norm_f16_index_order([&](int c) { return tile_chunk(st, row, c); });
                    }
                }
            }
            const bool ok = mbar_wait(tfull_bar(acc), aph, abort_flag, kErrEpilogue);
            if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform: tcgen05.ld is .aligned
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)acc * kAccStride;
            if constexpr (!kSketchOut) {
                // The MMA has finished reading the stage: hand it back to the producer.
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(stage));
                uint32_t wbits[8];
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    if (c < nw) {
                        uint32_t r0[32], r1[32];
                        tmem_ld_32x32b_x32(taddr + (uint32_t)c * 32u, r0);
                        if (c + 1 < nw) tmem_ld_32x32b_x32(taddr + (uint32_t)(c + 1) * 32u, r1);
                        tmem_ld_wait();
                        wbits[c] = pack_nonneg_bits(r0);
                        if (c + 1 < nw) wbits[c + 1] = pack_nonneg_bits(r1);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(acc));
                if (key < n_rows) {
                    if (ss == 0.0f) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) wbits[c] = 0xFFFFFFFFu;
                    }
                    uint32_t* dst = words + key * nw;
                    if ((nw & 3) == 0) {
#pragma unroll
                        for (int c = 0; c < 8; c += 4)
                            if (c < nw)
                                *reinterpret_cast<uint4*>(dst + c) =
                                    make_uint4(wbits[c], wbits[c + 1], wbits[c + 2], wbits[c + 3]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (c < nw) dst[c] = wbits[c];
                    }
                    if (!deferred) norms[key] = nbits;
                }
            } else {
                float* dst = sketch_out + key * m;
#pragma unroll 1
                for (int c = 0; c < nw; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(taddr + (uint32_t)c * 32u, r);
                    tmem_ld_wait();
                    if (key < n_rows) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(dst + c * 32 + j) =
                                make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                            __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(tempty_bar(acc));
                    mbar_arrive(empty_bar(stage));
                }
            }
        }
        if constexpr (!kSketchOut) {
            // The deferred norms, one key per epilogue thread, from global memory (rows
            // are 256 bytes, so 16-byte aligned).  The barrier over the 256 epilogue
            // threads makes every queued key visible; every epilogue warp reaches it,
            // also after leaving its loop early.
            asm volatile("bar.sync 1, 256;" ::: "memory");
            const int cnt = min(slow_count, kSlowCap);
            for (int i = (int)threadIdx.x - 64; i < cnt; i += 256) {
                const uint32_t key = slow_keys[i];
                const uint4* src = reinterpret_cast<const uint4*>(rows + (size_t)key * kDim);
                norms[key] = norm_f16_index_order([&](int c) { return __ldg(src + c); });
            }
        }
    }

    __syncwarp();  // reconverge warps 0 and 1, whose lane 0 ran the role loop alone
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// --------------------------------------------------------------------------------
// Host side
// --------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D fp16 tensor [rows][128], box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kDim * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// 2-D byte tensor [rows][128], box = 128 bytes x box_rows rows, 128-byte swizzle: each
// row lands as 128 bytes with its 16-byte chunks permuted by the row index mod 8, the
// layout the tensor cores read an MN-major 8-bit operand from.
bool make_u8_rows_map(CUtensorMap* map, const void* ptr, int64_t rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)128};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

size_t smem_bytes(int m) {
    return 1024 /* alignment slack */ + 2u * (size_t)m * 128u + (size_t)kStages * kTileBytes +
           8u * (2 * kStages + 6);
}

template <bool kSketchOut>
cudaError_t launch_mma(const uint16_t* rows, int64_t n_rows, const uint16_t* S, int m,
                       uint32_t* words, uint16_t* norms, float* sketch, cudaStream_t st) {
    CUtensorMap map_rows, map_s;
    if (!make_map(&map_rows, rows, n_rows, kBM)) return cudaErrorNotSupported;
    if (!make_map(&map_s, S, m, m)) return cudaErrorNotSupported;
    const size_t smem = smem_bytes(m);
    cudaError_t e = cudaFuncSetAttribute(qjl_mma_kernel<kSketchOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t n_tiles = (n_rows + kBM - 1) / kBM;
    const int64_t sms = device_sm_count();
    const int grid = (int)(n_tiles < sms ? n_tiles : sms);
    qjl_mma_kernel<kSketchOut><<<grid, kThreads, smem, st>>>(map_rows, map_s, rows, n_rows, m,
                                                             words, norms, sketch);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qjl_encode(const uint16_t* keys, int64_t n_keys, const uint16_t* S, int m,
                              uint32_t* words, uint16_t* norms, cudaStream_t st) {
    return launch_mma<false>(keys, n_keys, S, m, words, norms, nullptr, st);
}

cudaError_t launch_qjl_query_sketch(const uint16_t* q, int64_t n_q, const uint16_t* S, int m,
                                    float* v, cudaStream_t st) {
    return launch_mma<true>(q, n_q, S, m, nullptr, nullptr, v, st);
}

cudaError_t read_and_clear_device_error(uint32_t* code) {
    unsigned int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_kvq_device_error, sizeof(v));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_kvq_device_error, &zero, sizeof(zero));
    *code = v;
    return e;
}

}  // namespace kvq
