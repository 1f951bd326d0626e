// Attention-sink eviction over the compressed cache: per-token attention mass, the
// retained-token selection and the compaction of the cache to the retained tokens.
//
// Definition: "Q-TensorFormer" model card, section 6, Attention-Sink Dynamic Eviction:
// when the context exceeds the memory budget the retained set is the initial prompt
// sinks (|K_sink| = 4) plus the top-K tokens by attention mass sum_h sum_i alpha_{h,i,j}
// (query heads h, decode steps i).  Readings: the mass is accumulated per batch row over
// all query heads into a caller-owned buffer, one decode step at a time; equal masses
// are ordered by the smaller token index; the retained tokens keep their order.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

__device__ unsigned int g_evict_error = 0;

namespace {

enum : unsigned int { kErrGatherIndex = 0x301 };

constexpr int kMassTok = 32;    // tokens per CTA (one per lane)
constexpr int kMassGroups = 8;  // head groups per CTA (one per warp)

// mass[b][t] += sum_h 2^(score[b][h][t] * scale_log2 - M_bh) / L_bh.  A CTA covers 32
// tokens of one batch row: warp g sums heads g, g + 8, ... (loads down the head axis
// coalesced across the 32 tokens), then the 8 partial sums are added in a fixed order,
// so the result does not depend on scheduling.  Launched as a programmatic dependent
// of the merge kernel: it waits for it (and so for the decode kernel) before reading.
__global__ void __launch_bounds__(kMassTok * kMassGroups) attention_mass_kernel(
    const float* __restrict__ scores, const float* __restrict__ fin_ml, int B, int Hq, int T, float scale_log2,
    float* __restrict__ mass) {
    __shared__ float part[kMassGroups][kMassTok];
    dev::griddep_wait();
    const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
    const int t = blockIdx.x * kMassTok + lane;
    for (int b = blockIdx.y; b < B; b += gridDim.y) {
        float acc = 0.0f;
        if (t < T) {
            const float* sb = scores + (int64_t)b * Hq * T + t;
            const float* mlb = fin_ml + (int64_t)b * Hq * 2;
            int h = g;
            for (; h + 3 * kMassGroups < Hq; h += 4 * kMassGroups) {
                float x[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) x[k] = __ldcs(sb + (int64_t)(h + k * kMassGroups) * T);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 ml = __ldg(reinterpret_cast<const float2*>(mlb) + h + k * kMassGroups);
                    acc += exp2f(x[k] * scale_log2 - ml.x) / ml.y;
                }
            }
            for (; h < Hq; h += kMassGroups) {
                const float2 ml = __ldg(reinterpret_cast<const float2*>(mlb) + h);
                acc += exp2f(__ldcs(sb + (int64_t)h * T) * scale_log2 - ml.x) / ml.y;
            }
        }
        part[g][lane] = acc;
        __syncthreads();
        if (g == 0 && t < T) {
            float sum = part[0][lane];
#pragma unroll
            for (int k = 1; k < kMassGroups; ++k) sum += part[k][lane];
            mass[(int64_t)b * T + t] += sum;
        }
        __syncthreads();
    }
}

// Order-preserving image of a float as an unsigned integer (larger float -> larger
// key; -0 and +0 map to the same key).
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelSmemKeys = 48 * 1024;  // rows up to this many tokens keep their keys in shared memory

// Inclusive prefix sum over the CTA of one value per thread; *total receives the sum
// over the CTA.
__device__ __forceinline__ int block_inclusive_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += n;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    const int r = v + (warp > 0 ? warp_tot[warp - 1] : 0);
    *total = warp_tot[kSelWarps - 1];
    __syncthreads();  // warp_tot is reused by the next scan
    return r;
}

// One CTA per batch row.  Radix select (4 passes of 8 bits, most significant first) of
// the K-th largest key among tokens [n_sink, T), K = n_keep - n_sink; then one ordered
// pass writes the kept tokens in increasing order: the sinks, every token whose key is
// above the K-th largest, and the first (by index) `need` tokens whose key equals it.
// SMEM: the row's keys are computed once into shared memory (T <= kSelSmemKeys).
template <bool SMEM>
__global__ void __launch_bounds__(kSelThreads) evict_select_kernel(const float* __restrict__ mass, int T,
                                                                   int n_sink, int n_keep,
                                                                   int32_t* __restrict__ kept) {
    extern __shared__ uint32_t skeys[];
    __shared__ unsigned int hist[256];
    __shared__ int warp_tot[kSelWarps];
    __shared__ uint32_t sh_prefix;
    __shared__ int sh_need;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* mb = mass + (int64_t)blockIdx.x * T;
    int32_t* kb = kept + (int64_t)blockIdx.x * n_keep;
    const int K = n_keep - n_sink;
    const bool take_all = K >= T - n_sink;
    auto key = [&](int t) -> uint32_t { return SMEM ? skeys[t] : order_key(mb[t]); };
    if (SMEM && K > 0 && !take_all) {
        for (int t = n_sink + threadIdx.x; t < T; t += kSelThreads) skeys[t] = order_key(mb[t]);
    }
    uint32_t prefix = 0, mask = 0;
    int need = K;  // how many of the candidates equal to the selected prefix to take
    if (K > 0 && !take_all) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (threadIdx.x < 256) hist[threadIdx.x] = 0u;
            __syncthreads();
            for (int t0 = n_sink; t0 < T; t0 += kSelThreads) {
                const int t = t0 + threadIdx.x;
                bool hit = false;
                uint32_t digit = 0;
                if (t < T) {
                    const uint32_t k = key(t);
                    hit = (k & mask) == prefix;
                    digit = (k >> shift) & 0xFFu;
                }
                // one shared atomic per distinct digit of the warp (keys cluster heavily)
                const unsigned hits = __ballot_sync(0xffffffffu, hit);
                if (hit) {
                    const unsigned peers = __match_any_sync(hits, digit);
                    if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
                }
            }
            __syncthreads();
            // digit selection: thread i holds digit 255 - i; an inclusive scan in that
            // order gives the count of candidates at or above each digit, and the one
            // thread whose range holds the need-th candidate publishes the digit.
            int c = 0, incl = 0;
            if (threadIdx.x < 256) {
                c = (int)hist[255 - threadIdx.x];
                incl = c;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int n = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += n;
                }
                if (lane == 31) warp_tot[warp] = incl;
            }
            __syncthreads();
            if (threadIdx.x < 256) {
                for (int w = 0; w < warp; ++w) incl += warp_tot[w];
                if (incl - c < need && need <= incl) {
                    sh_need = need - (incl - c);
                    sh_prefix = prefix | ((uint32_t)(255 - threadIdx.x) << shift);
                }
            }
            __syncthreads();
            need = sh_need;
            prefix = sh_prefix;
            mask |= 0xFFu << shift;
        }
    }
    int out_base = 0, eq_base = 0;
    for (int t0 = 0; t0 < T; t0 += kSelThreads) {
        const int t = t0 + threadIdx.x;
        int is_eq = 0, keep = 0;
        if (t < T) {
            if (t < n_sink || take_all) {
                keep = 1;
            } else if (K > 0) {
                const uint32_t k = key(t);
                keep = k > prefix;
                is_eq = k == prefix;
            }
        }
        int eq_total, keep_total;
        const int eq_incl = block_inclusive_scan(is_eq, warp_tot, &eq_total);
        if (is_eq && eq_base + eq_incl <= need) keep = 1;
        const int keep_incl = block_inclusive_scan(keep, warp_tot, &keep_total);
        if (keep) kb[out_base + keep_incl - 1] = t;
        eq_base += eq_total;
        out_base += keep_total;
    }
}

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 8;  // pieces in flight per lane

// Warp-level copy of kGatherRows (32) consecutive kept rows (from j0) of one (b, h): one
// coalesced load of their indices, then the rows' UNIT pieces in lane order,
// kGatherUnroll loads in flight per lane before the stores (contiguous in dst).  A kept
// index outside [0, src_rows) is recorded in g_evict_error and that row is skipped.
// (64-row items with 16 pieces in flight measured slower on B200.)
constexpr int kGatherRows = 32;

template <typename UNIT>
__device__ __forceinline__ void gather_group(const UNIT* __restrict__ src, UNIT* __restrict__ dst, int64_t bh,
                                             int H, int64_t src_rows, int64_t dst_rows, int units, int ushift,
                                             const int32_t* __restrict__ kept, int n_keep, int j0, int lane) {
    const int nrows = min(kGatherRows, n_keep - j0);
    int32_t r_lane = -1;
    if (lane < nrows) {
        r_lane = __ldg(kept + (bh / H) * n_keep + j0 + lane);
        if (r_lane < 0 || r_lane >= src_rows) {
            atomicCAS(&g_evict_error, 0u, kErrGatherIndex);
            r_lane = -1;
        }
    }
    const UNIT* s = src + bh * src_rows * units;
    UNIT* d = dst + (bh * dst_rows + j0) * units;
    const int pieces = nrows * units;
    for (int p0 = 0; p0 < pieces; p0 += 32 * kGatherUnroll) {
        UNIT v[kGatherUnroll];
        bool ok[kGatherUnroll];
#pragma unroll
        for (int k = 0; k < kGatherUnroll; ++k) {
            const int p = p0 + k * 32 + lane;
            const int jj = p < pieces ? (ushift >= 0 ? (p >> ushift) : p / units) : 0;
            const int32_t r = __shfl_sync(0xffffffffu, r_lane, jj);
            ok[k] = p < pieces && r >= 0;
            if (ok[k]) v[k] = __ldcs(s + (int64_t)r * units + (p - jj * units));
        }
#pragma unroll
        for (int k = 0; k < kGatherUnroll; ++k)
            if (ok[k]) d[p0 + k * 32 + lane] = v[k];
    }
}

// Rows of a single UNIT (4-16 B): a warp item covers kGatherSmallRows (256) kept rows,
// a lane takes rows j0 + lane + 32 k with their 8 indices and 8 data loads in flight.
constexpr int kGatherSmallRows = 256;

template <typename UNIT>
__device__ __forceinline__ void gather_group_small(const UNIT* __restrict__ src, UNIT* __restrict__ dst, int64_t bh,
                                                   int H, int64_t src_rows, int64_t dst_rows,
                                                   const int32_t* __restrict__ kept, int n_keep, int j0, int lane) {
    constexpr int K = kGatherSmallRows / 32;
    const int32_t* kb = kept + (bh / H) * n_keep;
    const UNIT* s = src + bh * src_rows;
    UNIT* d = dst + bh * dst_rows;
    int32_t r[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const int j = j0 + lane + 32 * k;
        r[k] = j < n_keep ? __ldg(kb + j) : -1;
        if (j < n_keep && (r[k] < 0 || r[k] >= src_rows)) {
            atomicCAS(&g_evict_error, 0u, kErrGatherIndex);
            r[k] = -1;
        }
    }
    UNIT v[K];
#pragma unroll
    for (int k = 0; k < K; ++k)
        if (r[k] >= 0) v[k] = __ldcs(s + r[k]);
#pragma unroll
    for (int k = 0; k < K; ++k)
        if (r[k] >= 0) d[j0 + lane + 32 * k] = v[k];
}

// dst[bh][j] = src[bh][kept[b][j]] for rows of `units` UNITs, j < n_keep (bh = b * H + h):
// a warp per 32 kept rows of one (b, h).
template <typename UNIT>
__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(
    const UNIT* __restrict__ src, UNIT* __restrict__ dst, int64_t BH, int H, int64_t src_rows, int64_t dst_rows,
    int units, int ushift, const int32_t* __restrict__ kept, int n_keep) {
    const int lane = threadIdx.x & 31;
    const int rows_item = units == 1 ? kGatherSmallRows : kGatherRows;
    const int groups = (n_keep + rows_item - 1) / rows_item;
    const int64_t n_work = BH * groups;
    const int64_t n_warps = (int64_t)gridDim.x * (kGatherThreads / 32);
    for (int64_t w = (int64_t)blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5); w < n_work; w += n_warps) {
        const int64_t bh = w / groups;
        const int j0 = (int)(w - bh * groups) * rows_item;
        if (units == 1)
            gather_group_small<UNIT>(src, dst, bh, H, src_rows, dst_rows, kept, n_keep, j0, lane);
        else
            gather_group<UNIT>(src, dst, bh, H, src_rows, dst_rows, units, ushift, kept, n_keep, j0, lane);
    }
}

// Several arrays compacted in one launch: the warps walk the arrays' work items one
// array after another; each array moves in the widest unit its rows and bases allow.
constexpr int kMaxGatherArrays = 8;
struct GatherSet {
    const void* src[kMaxGatherArrays];
    void* dst[kMaxGatherArrays];
    int64_t src_rows[kMaxGatherArrays];
    int64_t dst_rows[kMaxGatherArrays];
    int64_t work_end[kMaxGatherArrays];   // cumulative warp work items
    int units[kMaxGatherArrays];
    int ushift[kMaxGatherArrays];
    int unit_bytes[kMaxGatherArrays];
    int rows_item[kMaxGatherArrays];      // kept rows per warp item
    int n;
};

__global__ void __launch_bounds__(kGatherThreads, 2) gather_multi_kernel(const GatherSet gs, int H,
                                                                      const int32_t* __restrict__ kept, int n_keep) {
    const int lane = threadIdx.x & 31;
    const int64_t n_work = gs.work_end[gs.n - 1];
    const int64_t n_warps = (int64_t)gridDim.x * (kGatherThreads / 32);
    for (int64_t w = (int64_t)blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5); w < n_work; w += n_warps) {
        int a = 0;
        while (a + 1 < gs.n && w >= gs.work_end[a]) ++a;
        const int64_t local = w - (a > 0 ? gs.work_end[a - 1] : 0);
        const int rows_item = gs.rows_item[a];
        const int groups = (n_keep + rows_item - 1) / rows_item;
        const int64_t bh = local / groups;
        const int j0 = (int)(local - bh * groups) * rows_item;
        if (gs.units[a] == 1) {
            switch (gs.unit_bytes[a]) {
                case 16:
                    gather_group_small<uint4>(static_cast<const uint4*>(gs.src[a]), static_cast<uint4*>(gs.dst[a]), bh,
                                              H, gs.src_rows[a], gs.dst_rows[a], kept, n_keep, j0, lane);
                    break;
                case 4:
                    gather_group_small<uint32_t>(static_cast<const uint32_t*>(gs.src[a]),
                                                 static_cast<uint32_t*>(gs.dst[a]), bh, H, gs.src_rows[a],
                                                 gs.dst_rows[a], kept, n_keep, j0, lane);
                    break;
                case 2:
                    gather_group_small<uint16_t>(static_cast<const uint16_t*>(gs.src[a]),
                                                 static_cast<uint16_t*>(gs.dst[a]), bh, H, gs.src_rows[a],
                                                 gs.dst_rows[a], kept, n_keep, j0, lane);
                    break;
                default:
                    gather_group_small<uint8_t>(static_cast<const uint8_t*>(gs.src[a]), static_cast<uint8_t*>(gs.dst[a]),
                                                bh, H, gs.src_rows[a], gs.dst_rows[a], kept, n_keep, j0, lane);
            }
            continue;
        }
        switch (gs.unit_bytes[a]) {
            case 16:
                gather_group<uint4>(static_cast<const uint4*>(gs.src[a]), static_cast<uint4*>(gs.dst[a]), bh, H,
                                    gs.src_rows[a], gs.dst_rows[a], gs.units[a], gs.ushift[a], kept, n_keep, j0, lane);
                break;
            case 4:
                gather_group<uint32_t>(static_cast<const uint32_t*>(gs.src[a]), static_cast<uint32_t*>(gs.dst[a]), bh,
                                       H, gs.src_rows[a], gs.dst_rows[a], gs.units[a], gs.ushift[a], kept, n_keep, j0,
                                       lane);
                break;
            case 2:
                gather_group<uint16_t>(static_cast<const uint16_t*>(gs.src[a]), static_cast<uint16_t*>(gs.dst[a]), bh,
                                       H, gs.src_rows[a], gs.dst_rows[a], gs.units[a], gs.ushift[a], kept, n_keep, j0,
                                       lane);
                break;
            default:
                gather_group<uint8_t>(static_cast<const uint8_t*>(gs.src[a]), static_cast<uint8_t*>(gs.dst[a]), bh, H,
                                      gs.src_rows[a], gs.dst_rows[a], gs.units[a], gs.ushift[a], kept, n_keep, j0,
                                      lane);
        }
    }
}

}  // namespace

cudaError_t launch_attention_mass(const float* scores, const float* fin_ml, int64_t B, int64_t Hq,
                                  int64_t T, float scale_log2, float* mass, cudaStream_t st) {
    if (B * T == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((T + kMassTok - 1) / kMassTok), (unsigned)(B < 65535 ? B : 65535));
    cfg.blockDim = dim3(kMassTok * kMassGroups);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attention_mass_kernel, scores, fin_ml, (int)B, (int)Hq, (int)T, scale_log2,
                              mass);
}

cudaError_t launch_evict_select(const float* mass, int64_t B, int64_t T, int64_t n_sink, int64_t n_keep,
                                int32_t* kept, cudaStream_t st) {
    if (B == 0 || n_keep == 0) return cudaSuccess;
    if (T <= kSelSmemKeys) {
        const cudaError_t e = cudaFuncSetAttribute(
            evict_select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelSmemKeys * (int)sizeof(uint32_t));
        if (e != cudaSuccess) return e;
        const size_t smem = (size_t)T * sizeof(uint32_t);
        evict_select_kernel<true><<<(unsigned)B, kSelThreads, smem, st>>>(mass, (int)T, (int)n_sink, (int)n_keep,
                                                                           kept);
    } else {
        evict_select_kernel<false><<<(unsigned)B, kSelThreads, 0, st>>>(mass, (int)T, (int)n_sink, (int)n_keep,
                                                                         kept);
    }
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, void* dst, int64_t B, int64_t H, int64_t src_rows,
                               int64_t dst_rows, int64_t row_bytes, const int32_t* kept, int64_t n_keep,
                               cudaStream_t st) {
    const int64_t BH = B * H;
    if (BH == 0 || n_keep == 0) return cudaSuccess;
    // the widest unit that divides the row and both base addresses
    const uintptr_t al = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) | (uintptr_t)row_bytes;
    const int ub = (al % 16 == 0) ? 16 : (al % 4 == 0) ? 4 : (al % 2 == 0) ? 2 : 1;
    const int units = (int)(row_bytes / ub);
    const int ushift = (units & (units - 1)) == 0 ? __builtin_ctz((unsigned)units) : -1;
    const int64_t rows_item = (row_bytes / ub == 1) ? kGatherSmallRows : kGatherRows;
    const int64_t work = BH * ((n_keep + rows_item - 1) / rows_item);  // warps' units of work
    const int64_t want = (work + kGatherThreads / 32 - 1) / (kGatherThreads / 32);
    const int64_t cap = (int64_t)device_sm_count() * 16;  // about 4 waves of 4 resident CTAs
    dim3 grid((unsigned)(want < cap ? want : cap));
    const int Hi = (int)H, nk = (int)n_keep;
    switch (ub) {
        case 16:
            gather_rows_kernel<uint4><<<grid, kGatherThreads, 0, st>>>(
                static_cast<const uint4*>(src), static_cast<uint4*>(dst), BH, Hi, src_rows, dst_rows, units, ushift,
                kept, nk);
            break;
        case 4:
            gather_rows_kernel<uint32_t><<<grid, kGatherThreads, 0, st>>>(
                static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), BH, Hi, src_rows, dst_rows, units,
                ushift, kept, nk);
            break;
        case 2:
            gather_rows_kernel<uint16_t><<<grid, kGatherThreads, 0, st>>>(
                static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), BH, Hi, src_rows, dst_rows, units,
                ushift, kept, nk);
            break;
        default:
            gather_rows_kernel<uint8_t><<<grid, kGatherThreads, 0, st>>>(
                static_cast<const uint8_t*>(src), static_cast<uint8_t*>(dst), BH, Hi, src_rows, dst_rows, units,
                ushift, kept, nk);
    }
    return cudaGetLastError();
}

cudaError_t launch_gather_rows_multi(const GatherArray* arrays, int n_arrays, int64_t B, int64_t H,
                                     const int32_t* kept, int64_t n_keep, cudaStream_t st) {
    const int64_t BH = B * H;
    if (BH == 0 || n_keep == 0 || n_arrays == 0) return cudaSuccess;
    if (n_arrays > kMaxGatherArrays) return cudaErrorInvalidValue;
    GatherSet gs{};
    gs.n = n_arrays;
    // arrays with short rows first: their warps wait mostly on the index and data
    // latency, which the long-row arrays' streaming then overlaps
    int order[kMaxGatherArrays];
    for (int a = 0; a < n_arrays; ++a) order[a] = a;
    for (int a = 1; a < n_arrays; ++a)
        for (int b = a; b > 0 && arrays[order[b]].row_bytes < arrays[order[b - 1]].row_bytes; --b) {
            const int t = order[b];
            order[b] = order[b - 1];
            order[b - 1] = t;
        }
    int64_t acc = 0;
    for (int a = 0; a < n_arrays; ++a) {
        const GatherArray& g = arrays[order[a]];
        const uintptr_t al = reinterpret_cast<uintptr_t>(g.src) | reinterpret_cast<uintptr_t>(g.dst) |
                             (uintptr_t)g.row_bytes;
        const int ub = (al % 16 == 0) ? 16 : (al % 4 == 0) ? 4 : (al % 2 == 0) ? 2 : 1;
        const int units = (int)(g.row_bytes / ub);
        gs.src[a] = g.src;
        gs.dst[a] = g.dst;
        gs.src_rows[a] = g.src_rows;
        gs.dst_rows[a] = g.dst_rows;
        gs.units[a] = units;
        gs.ushift[a] = (units & (units - 1)) == 0 ? __builtin_ctz((unsigned)units) : -1;
        gs.unit_bytes[a] = ub;
        gs.rows_item[a] = units == 1 ? kGatherSmallRows : kGatherRows;
        acc += BH * ((n_keep + gs.rows_item[a] - 1) / gs.rows_item[a]);
        gs.work_end[a] = acc;
    }
    const int64_t want = (acc + kGatherThreads / 32 - 1) / (kGatherThreads / 32);
    const int64_t cap = (int64_t)device_sm_count() * 16;
    gather_multi_kernel<<<(unsigned)(want < cap ? want : cap), kGatherThreads, 0, st>>>(gs, (int)H, kept, (int)n_keep);
    return cudaGetLastError();
}

cudaError_t read_and_clear_evict_error(uint32_t* code) {
    unsigned int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_evict_error, sizeof(v));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_evict_error, &zero, sizeof(zero));
    *code = v;
    return e;
}

}  // namespace kvq
