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

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kCodeMagic = 12583040.0f;  // 1.5 * 2^23 + 128

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

// ---- packed fp32x2 arithmetic (sm_100): one instruction for two lanes of a pair ----
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
    float2 f;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
    return f;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Four int8 codes (one word, each byte biased by 128) -> two exact float pairs.
__device__ __forceinline__ void codes4(uint32_t biased, uint64_t& c01, uint64_t& c23) {
    const uint64_t magic = pack2(-kCodeMagic, -kCodeMagic);
    const float f0 = __uint_as_float(__byte_perm(biased, 0x4B400000u, 0x7650u));
    const float f1 = __uint_as_float(__byte_perm(biased, 0x4B400000u, 0x7651u));
    const float f2 = __uint_as_float(__byte_perm(biased, 0x4B400000u, 0x7652u));
    const float f3 = __uint_as_float(__byte_perm(biased, 0x4B400000u, 0x7653u));
    c01 = add2(pack2(f0, f1), magic);
    c23 = add2(pack2(f2, f3), magic);
}

// Max over the warp of a float (monotone map to int, then redux.sync).
__device__ __forceinline__ float warp_max(float v) {
    int i = __float_as_int(v);
    i = i >= 0 ? i : (i ^ 0x7FFFFFFF);
    i = __reduce_max_sync(0xffffffffu, i);
    return __int_as_float(i >= 0 ? i : (i ^ 0x7FFFFFFF));
}

// Merge of per-warp softmax states (m, l, acc[D]) through shared memory into the
// split's partial slot.  red: [WARPS][G][2 + kD] floats, already written.
template <int G, int WARPS>
__device__ __forceinline__ void merge_warps_and_store_n(const float* red, const DecodeParams& p,
                                                        int64_t unit, int split, int nthreads) {
    for (int idx = threadIdx.x; idx < G * kD; idx += nthreads) {
        const int g = idx / kD;
        const int d = idx % kD;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) mx = fmaxf(mx, red[(w * G + g) * (2 + kD)]);
        float l = 0.0f, a = 0.0f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float* r = red + (w * G + g) * (2 + kD);
            const float f = mx == -INFINITY ? 0.0f : exp2f(r[0] - mx);
            l += r[1] * f;
            a += r[2 + d] * f;
        }
        const int64_t slot = (unit * G + g) * p.splits + split;
        p.ws_acc[slot * kD + d] = a;
        if (d == 0) {
            p.ws_ml[slot * 2] = mx;
            p.ws_ml[slot * 2 + 1] = l;
        }
    }
}

// -----------------------------------------------------------------------------------
// INT8 keys.  The CTA's token chunk streams through a 4-stage shared-memory ring of
// 64-token stages (K rows and V rows, 8 KB each) filled by bulk asynchronous copies
// that one producer thread issues; eight consumer warps read the stage from shared
// memory.  8 lanes share a token (lane `sub` owns dims 16 sub .. 16 sub + 15 of K and
// V); each 8-lane group takes 2 consecutive tokens of the stage and keeps its own
// online-softmax state, merged across groups (shuffles) and warps (shared memory) at
// the end.  Scales are read with ordinary loads issued before the stage wait.
// -----------------------------------------------------------------------------------
constexpr int kI8StageTok = 64;
constexpr int kI8Stages = 4;
constexpr int kI8StageBytes = 2 * kI8StageTok * kD;    // K rows then V rows

__device__ unsigned int g_decode_error = 0;

enum : unsigned int { kErrI8Producer = 0x201, kErrI8Consumer = 0x202 };

constexpr int kI8Consumers = 8;                          // consumer warps; warp 8 produces
constexpr int kI8Threads = 32 * (kI8Consumers + 1);

template <int G>
__global__ void __launch_bounds__(kI8Threads)
decode_int8_kernel(const DecodeParams p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ uint64_t bars[2 * kI8Stages];
    __shared__ int abort_storage;
    volatile int* abort_flag = &abort_storage;
    constexpr int U = kI8StageTok / (kI8Consumers * 4);   // tokens per 8-lane group per stage
    const int64_t unit = blockIdx.x;
    const int split = blockIdx.y;
    const int64_t b = unit / p.Hkv;
    const int kvh = (int)(unit % p.Hkv);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t T = p.T;
    const int64_t t_begin = (int64_t)split * p.chunk;
    const int64_t t_end = min(T, t_begin + p.chunk);
    const int64_t row0 = unit * T;
    const int n_steps = (int)((t_end - t_begin + kI8StageTok - 1) / kI8StageTok);
    const uint32_t ring = dev::smem_u32(smem_raw);
    const uint32_t bar0 = dev::smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kI8Stages + s); };

    if (threadIdx.x == 0) {
        abort_storage = 0;
        for (int s = 0; s < kI8Stages; ++s) {
            dev::mbar_init(full_bar(s), 1);
            dev::mbar_init(empty_bar(s), kI8Consumers);
        }
        dev::mbar_init_fence();
    }
    __syncthreads();

    if (warp == kI8Consumers) {
        // ---------------- producer ----------------
        if (lane == 0) {
            bool issued[kI8Stages] = {false, false, false, false};
            uint32_t ph_issued[kI8Stages] = {0, 0, 0, 0};
            for (int i = 0; i < n_steps; ++i) {
                const int s = i % kI8Stages;
                const uint32_t ph = (uint32_t)(i / kI8Stages) & 1u;
                if (!dev::mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, &g_decode_error, kErrI8Producer)) break;
                const int64_t t = t_begin + (int64_t)i * kI8StageTok;
                const uint32_t n = (uint32_t)min((int64_t)kI8StageTok, t_end - t);
                const uint32_t dst = ring + (uint32_t)s * kI8StageBytes;
                // Values are copied only when the output is wanted (scores-only calls pass
                // no value pointers).
                dev::mbar_arrive_expect_tx(full_bar(s), (p.want_out ? 2u : 1u) * n * kD);
                dev::bulk_g2s(dst, p.kc + (row0 + t) * kD, n * kD, full_bar(s));
                if (p.want_out)
                    dev::bulk_g2s(dst + kI8StageTok * kD, p.vc + (row0 + t) * kD, n * kD, full_bar(s));
                issued[s] = true;
                ph_issued[s] = ph;
            }
            for (int s = 0; s < kI8Stages; ++s)
                if (issued[s]) dev::mbar_drain(full_bar(s), ph_issued[s]);
        }
        __syncwarp();
        __syncthreads();  // matches the consumers' barrier before the merge
        return;
    }

    // ---------------- consumers (warps 0 .. kI8Consumers-1) ----------------
    const int tg = lane >> 3;
    const int sub = lane & 7;
    uint64_t qp[G][8];
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
            qp[g][i] = pack2(f0.x, f0.y);
            qp[g][4 + i] = pack2(f1.x, f1.y);
        }
    }
    float mrun[G], lrun[G];
    uint64_t acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        mrun[g] = -INFINITY;
        lrun[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[g][i] = 0ull;
    }

    for (int i = 0; i < n_steps; ++i) {
        const int s = i % kI8Stages;
        const uint32_t ph = (uint32_t)(i / kI8Stages) & 1u;
        const int64_t tstage = t_begin + (int64_t)i * kI8StageTok;
        const int tok0 = warp * (4 * U) + tg * U;        // first token of this group in the stage
        bool valid[U];
        float ksc[U], vsc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t t = tstage + tok0 + u;
            valid[u] = t < t_end;
            const int64_t r = row0 + (valid[u] ? t : t_begin);
            ksc[u] = __ldg(p.ks + r);
            vsc[u] = p.want_out ? __ldg(p.vs + r) : 0.0f;
        }
        const bool ok = dev::mbar_wait(full_bar(s), ph, abort_flag, &g_decode_error, kErrI8Consumer);
        if (!__all_sync(0xffffffffu, ok)) break;
        const unsigned char* kst = smem_raw + (size_t)s * kI8StageBytes;
        const unsigned char* vst = kst + kI8StageTok * kD;
        float score[U][G];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint4 kv = *reinterpret_cast<const uint4*>(kst + (tok0 + u) * kD + sub * 16);
            uint64_t c[8];
            const uint32_t w4[4] = {kv.x ^ 0x80808080u, kv.y ^ 0x80808080u, kv.z ^ 0x80808080u,
                                    kv.w ^ 0x80808080u};
#pragma unroll
            for (int q = 0; q < 4; ++q) codes4(w4[q], c[2 * q], c[2 * q + 1]);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                uint64_t dp0 = 0ull, dp1 = 0ull;
#pragma unroll
                for (int q = 0; q < 8; q += 2) {
                    dp0 = fma2(qp[g][q], c[q], dp0);
                    dp1 = fma2(qp[g][q + 1], c[q + 1], dp1);
                }
                const float2 d2 = unpack2(add2(dp0, dp1));
                float d = d2.x + d2.y;
                d += __shfl_xor_sync(0xffffffffu, d, 1);
                d += __shfl_xor_sync(0xffffffffu, d, 2);
                d += __shfl_xor_sync(0xffffffffu, d, 4);
                score[u][g] = d * ksc[u];
            }
        }
        if (p.scores_out != nullptr && sub == 0) {
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (valid[u]) {
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        p.scores_out[(b * p.Hq + (int64_t)kvh * G + g) * T + tstage + tok0 + u] = score[u][g];
                }
        }
        if (p.want_out) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float mb = -INFINITY;
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (valid[u]) mb = fmaxf(mb, score[u][g] * p.scale_log2);
                if (mb > mrun[g]) {
                    const float corr = exp2f(mrun[g] - mb);
                    lrun[g] *= corr;
                    const uint64_t c2 = pack2(corr, corr);
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[g][q] = mul2(acc[g][q], c2);
                    mrun[g] = mb;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!valid[u]) continue;
                const uint4 vv = *reinterpret_cast<const uint4*>(vst + (tok0 + u) * kD + sub * 16);
                uint64_t c[8];
                const uint32_t w4[4] = {vv.x ^ 0x80808080u, vv.y ^ 0x80808080u, vv.z ^ 0x80808080u,
                                        vv.w ^ 0x80808080u};
#pragma unroll
                for (int q = 0; q < 4; ++q) codes4(w4[q], c[2 * q], c[2 * q + 1]);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float pe = exp2f(score[u][g] * p.scale_log2 - mrun[g]);
                    lrun[g] += pe;
                    const float wv = pe * vsc[u];
                    const uint64_t w2 = pack2(wv, wv);
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[g][q] = fma2(w2, c[q], acc[g][q]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(empty_bar(s));
    }

    // merge the 4 lane groups of each warp (lanes l, l^8, l^16, l^24)
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
            for (int q = 0; q < 8; ++q) {
                const float2 a = unpack2(acc[g][q]);
                const float ax = __shfl_xor_sync(0xffffffffu, a.x, off);
                const float ay = __shfl_xor_sync(0xffffffffu, a.y, off);
                acc[g][q] = pack2(a.x * f1 + ax * f2, a.y * f1 + ay * f2);
            }
            mrun[g] = mn;
        }
    }
    // All stages are consumed (or the CTA aborted): reuse the ring for the merge.
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kI8Consumers) : "memory");
    float* red = reinterpret_cast<float*>(smem_raw);  // [consumer warps][G][2 + kD]
    if (p.want_out && tg == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float* r = red + (warp * G + g) * (2 + kD);
            if (sub == 0) {
                r[0] = mrun[g];
                r[1] = lrun[g];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float2 a = unpack2(acc[g][q]);
                r[2 + sub * 16 + 2 * q] = a.x;
                r[2 + sub * 16 + 2 * q + 1] = a.y;
            }
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kI8Consumers) : "memory");
    if (p.want_out) merge_warps_and_store_n<G, kI8Consumers>(red, p, unit, split, 32 * kI8Consumers);
    __syncthreads();  // matches the producer warp's final barrier
}

// -----------------------------------------------------------------------------------
// QJL keys.  A warp takes 32 tokens per step.
//  * Byte tables: LUT[p][b] (G floats) = sum_{k<8} v_g[8p + k] * (bit k of b ? +1 : -1),
//    stored as two halves of 16 positions, entry (p, b) at
//    (p / 16) * 64 KB + b * 256 B + (p % 16) * 16 B.  Thread (p, c) fills the 16 bytes
//    b = 16c .. 16c+15 of position p: one 8-term sum, then 15 steps along a Gray code
//    of the low nibble (one add per step), 16-byte stores contiguous across lanes.
//  * Scores: lane l scores token t0 + l from its 32 bytes of sign words, 32 lookups.
//    Lane l visits the 8 byte positions of each 64-bit word pair in the order e ^ (l & 7),
//    so at every step the 8 lanes of each quarter-warp read 8 different 16-byte bank
//    groups (a 512-byte LDS.128 in the minimum 4 wavefronts).  One byte permute builds
//    each lookup's offset: the selected sign byte lands in bits 8..15 next to the lane's
//    (e ^ (l & 7)) * 16 in bits 0..7.
//  * Softmax: warp-wide running max per head (redux.sync on an order-preserving int
//    image), per-lane running sums.
//  * Values: the weights w = p * v_scale go through shared memory interleaved by token
//    pairs; lane l owns dims 4l .. 4l+3 of every token's value row (one 4-byte load per
//    token, a contiguous 128-byte row across the warp) and keeps (even token, odd token)
//    partial sums in packed fp32x2 registers, so each fp32x2 FMA consumes a weight pair
//    and a code pair as they come.
// -----------------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(512, 1)
decode_qjl_kernel(const DecodeParams p) {
    extern __shared__ float4 dsmem4[];
    float* dsmem = reinterpret_cast<float*>(dsmem4);
    constexpr int THREADS = 512;
    constexpr int WARPS = THREADS / 32;
    constexpr int TOK_PER_STEP = WARPS * 32;
    constexpr int HALF_FLOATS = 256 * 16 * 4;        // one table half: 64 KB
    const int64_t unit = blockIdx.x;
    const int split = blockIdx.y;
    const int64_t b = unit / p.Hkv;
    const int kvh = (int)(unit % p.Hkv);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t T = p.T;
    const int64_t t_begin = (int64_t)split * p.chunk;
    const int64_t t_end = min(T, t_begin + p.chunk);
    const int64_t row0 = unit * T;
    const int nw = p.m / 32;
    const int npos = p.m / 8;

    float* lut = dsmem;                              // 2 halves x [256][16] x 4 floats
    float* wbuf = dsmem + 2 * HALF_FLOATS;           // [WARPS][16 pairs][G][2]

    // ---- byte tables ----
    {
        const int pos = threadIdx.x & 31;
        const int c = threadIdx.x >> 5;               // high nibble of the byte value
        float v[G][8];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float* src = p.sketch_v + (b * p.Hq + (int64_t)kvh * G + g) * p.m + pos * 8;
#pragma unroll
            for (int k = 0; k < 8; ++k) v[g][k] = pos < npos ? __ldg(src + k) : 0.0f;
        }
        float val[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float s = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) s -= v[g][k];
#pragma unroll
            for (int k = 0; k < 4; ++k) s += ((c >> k) & 1) ? v[g][4 + k] : -v[g][4 + k];
            val[g] = s;
        }
        float* base = lut + (pos >> 4) * HALF_FLOATS + (c * 16 * 16 + (pos & 15)) * 4;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int gray = i ^ (i >> 1);
            if (i > 0) {
                const int k = __ffs(i) - 1;               // the bit that flips at step i
                const bool on = (gray >> k) & 1;
#pragma unroll
                for (int g = 0; g < G; ++g) val[g] += on ? 2.0f * v[g][k] : -2.0f * v[g][k];
            }
            float* e = base + gray * 16 * 4;              // byte 16c + gray: +gray*256 B
            *reinterpret_cast<float4*>(e) = make_float4(val[0], G > 1 ? val[G > 1 ? 1 : 0] : 0.0f,
                                                        G > 2 ? val[G > 2 ? 2 : 0] : 0.0f,
                                                        G > 3 ? val[G > 3 ? 3 : 0] : 0.0f);
        }
    }
    __syncthreads();

    const int x = lane & 7;
    const bool swap_words = (x & 4) != 0;
    // per step e: the lane's offset (e ^ x) * 16 in byte 0, and the permute selector that
    // puts byte ((e ^ x) & 3) of the chosen word in byte 1 and zeros in bytes 2, 3
    uint32_t off16[8];
    uint32_t sel[4];
#pragma unroll
    for (int e = 0; e < 8; ++e) off16[e] = (uint32_t)((e ^ x) * 16);
#pragma unroll
    for (int e = 0; e < 4; ++e) sel[e] = 0x6504u | ((uint32_t)((e ^ x) & 3) << 4);
    const uint32_t lut_s = (uint32_t)__cvta_generic_to_shared(lut);

    float mrun[G], lsum[G];
    uint64_t acc[G][4];                               // (even, odd) token partial sums, 4 dims
#pragma unroll
    for (int g = 0; g < G; ++g) {
        mrun[g] = -INFINITY;
        lsum[g] = 0.0f;
#pragma unroll
        for (int d = 0; d < 4; ++d) acc[g][d] = 0ull;
    }
    float* mybuf = wbuf + warp * 32 * G;
    const uint64_t magic = pack2(-kCodeMagic, -kCodeMagic);

    for (int64_t t0 = t_begin + (int64_t)warp * 32; t0 < t_end; t0 += TOK_PER_STEP) {
        const int nvalid = (int)min((int64_t)32, t_end - t0);
        const bool valid = lane < nvalid;
        const int64_t r = row0 + t0 + (valid ? lane : 0);
        // ---- loads: this lane's token (words, norm, value scale), and 4 value codes
        //      of each of the step's tokens ----
        uint32_t w[8];
        if (nw == 8) {
            const uint4 a = __ldcs(reinterpret_cast<const uint4*>(p.kw + r * 8));
            const uint4 c = __ldcs(reinterpret_cast<const uint4*>(p.kw + r * 8) + 1);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
            w[4] = c.x; w[5] = c.y; w[6] = c.z; w[7] = c.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = i < nw ? __ldcs(p.kw + r * nw + i) : 0u;
        }
        const float nrm = __half2float(__ushort_as_half(__ldcs(p.kn + r)));
        float vsc = 0.0f;
        uint32_t vcode[32];
        if (p.want_out) {
            vsc = __ldcs(p.vs + r);
            const unsigned int* vrow = reinterpret_cast<const unsigned int*>(p.vc + (row0 + t0) * kD) + lane;
#pragma unroll
            for (int j = 0; j < 32; ++j) vcode[j] = j < nvalid ? __ldcs(vrow + j * (kD / 4)) : 0x80808080u;
        }
        // ---- estimator: 32 byte-table lookups ----
        float sc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) sc[g] = 0.0f;
        uint64_t s01 = 0ull, s23 = 0ull;
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
            const uint32_t wa = swap_words ? w[2 * pr + 1] : w[2 * pr];
            const uint32_t wb = swap_words ? w[2 * pr] : w[2 * pr + 1];
            const uint32_t half_off = (uint32_t)((pr >> 1) * HALF_FLOATS * 4 + (pr & 1) * 128);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t o = __byte_perm(e < 4 ? wa : wb, off16[e], sel[e & 3]);
                const uint32_t addr = lut_s + half_off + o;
                if constexpr (G == 4) {
                    float4 f;
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(f.x), "=f"(f.y), "=f"(f.z), "=f"(f.w) : "r"(addr));
                    s01 = add2(s01, pack2(f.x, f.y));
                    s23 = add2(s23, pack2(f.z, f.w));
                } else if constexpr (G == 2) {
                    float2 f;
                    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(f.x), "=f"(f.y) : "r"(addr));
                    s01 = add2(s01, pack2(f.x, f.y));
                } else {
                    float f;
                    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f) : "r"(addr));
                    sc[0] += f;
                }
            }
        }
        if constexpr (G >= 2) {
            const float2 a = unpack2(s01);
            sc[0] = a.x;
            sc[1] = a.y;
        }
        if constexpr (G == 4) {
            const float2 a = unpack2(s23);
            sc[2] = a.x;
            sc[3] = a.y;
        }
        float score[G];
#pragma unroll
        for (int g = 0; g < G; ++g) score[g] = p.qjl_c * nrm * sc[g];
        if (p.scores_out != nullptr && valid) {
#pragma unroll
            for (int g = 0; g < G; ++g)
                p.scores_out[(b * p.Hq + (int64_t)kvh * G + g) * T + t0 + lane] = score[g];
        }
        if (!p.want_out) continue;
        // ---- online softmax at warp granularity ----
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float lg = valid ? score[g] * p.scale_log2 : -INFINITY;
            const float mb = warp_max(lg);
            if (mb > mrun[g]) {
                const float corr = exp2f(mrun[g] - mb);
                lsum[g] *= corr;
                const uint64_t c2 = pack2(corr, corr);
#pragma unroll
                for (int d = 0; d < 4; ++d) acc[g][d] = mul2(acc[g][d], c2);
                mrun[g] = mb;
            }
            const float pe = exp2f(lg - mrun[g]);
            lsum[g] += pe;
            mybuf[(lane >> 1) * (2 * G) + g * 2 + (lane & 1)] = pe * vsc;
        }
        __syncwarp();
        // ---- values: dims 4 lane .. 4 lane + 3, token pairs (2 jp, 2 jp + 1) ----
#pragma unroll
        for (int jp = 0; jp < 16; ++jp) {
            const uint32_t ce = vcode[2 * jp] ^ 0x80808080u;
            const uint32_t co = vcode[2 * jp + 1] ^ 0x80808080u;
            uint64_t cp[4];
#pragma unroll
            for (int d = 0; d < 4; ++d)
                cp[d] = add2(pack2(__uint_as_float(__byte_perm(ce, 0x4B400000u, 0x7650u + d)),
                                   __uint_as_float(__byte_perm(co, 0x4B400000u, 0x7650u + d))),
                             magic);
            uint64_t wp[G];
            if constexpr (G == 4) {
                const float4 a = reinterpret_cast<const float4*>(mybuf)[jp * 2];
                const float4 c = reinterpret_cast<const float4*>(mybuf)[jp * 2 + 1];
                wp[0] = pack2(a.x, a.y); wp[1] = pack2(a.z, a.w);
                wp[2] = pack2(c.x, c.y); wp[3] = pack2(c.z, c.w);
            } else if constexpr (G == 2) {
                const float4 a = reinterpret_cast<const float4*>(mybuf)[jp];
                wp[0] = pack2(a.x, a.y); wp[1] = pack2(a.z, a.w);
            } else {
                const float2 a = reinterpret_cast<const float2*>(mybuf)[jp];
                wp[0] = pack2(a.x, a.y);
            }
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int d = 0; d < 4; ++d) acc[g][d] = fma2(wp[g], cp[d], acc[g][d]);
        }
        __syncwarp();
    }
    if (!p.want_out) return;

    // ---- per-warp state -> shared memory -> merged split state ----
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], off);
    __syncthreads();  // the byte tables are no longer read
    float* red = dsmem;  // [WARPS][G][2 + kD]
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float* rr = red + (warp * G + g) * (2 + kD);
        if (lane == 0) {
            rr[0] = mrun[g];
            rr[1] = lsum[g];
        }
#pragma unroll
        for (int d = 0; d < 4; ++d) {
            const float2 a = unpack2(acc[g][d]);
            rr[2 + 4 * lane + d] = a.x + a.y;
        }
    }
    __syncthreads();
    merge_warps_and_store_n<G, WARPS>(red, p, unit, split, WARPS * 32);
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

constexpr int kInt8TokPerStep = kI8StageTok;
constexpr int kQjlTokPerStep = 16 * 32;                // 16 warps x 32 tokens

template <int G>
size_t int8_smem() {
    const size_t ring = (size_t)kI8Stages * kI8StageBytes;
    const size_t red = (size_t)kI8Consumers * G * (2 + kD) * sizeof(float);
    return ring > red ? ring : red;
}
template <int G>
size_t qjl_smem() {
    const size_t tables = (size_t)2 * 256 * 16 * 4 * sizeof(float);   // entries padded to 16 B
    const size_t wbuf = (size_t)16 * 32 * G * sizeof(float);
    const size_t red = (size_t)16 * G * (2 + kD) * sizeof(float);
    const size_t a = tables + wbuf;
    return a > red ? a : red;
}

template <int G>
cudaError_t run_int8(const DecodeParams& p, int64_t units, cudaStream_t st) {
    auto kern = decode_int8_kernel<G>;
    const size_t smem = int8_smem<G>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)units, (unsigned)p.splits);
    kern<<<grid, kI8Threads, smem, st>>>(p);
    return cudaGetLastError();
}

template <int G>
cudaError_t run_qjl(const DecodeParams& p, int64_t units, cudaStream_t st) {
    auto kern = decode_qjl_kernel<G>;
    const size_t smem = qjl_smem<G>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)units, (unsigned)p.splits);
    kern<<<grid, 512, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t run_partial(bool qjl, int G, const DecodeParams& p, int64_t units, cudaStream_t st) {
    if (qjl) {
        switch (G) {
            case 1: return run_qjl<1>(p, units, st);
            case 2: return run_qjl<2>(p, units, st);
            case 4: return run_qjl<4>(p, units, st);
            default: return cudaErrorNotSupported;
        }
    }
    switch (G) {
        case 1: return run_int8<1>(p, units, st);
        case 2: return run_int8<2>(p, units, st);
        case 4: return run_int8<4>(p, units, st);
        case 8: return run_int8<8>(p, units, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t read_and_clear_decode_error(uint32_t* code) {
    unsigned int v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_decode_error, sizeof(v));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(zero));
    *code = v;
    return e;
}

DecodePlan plan_decode(const kvq_decode_args* a, int sm_count) {
    DecodePlan pl{};
    const int64_t G = a->n_q_heads / a->n_kv_heads;
    pl.units = a->batch * a->n_kv_heads;
    const int64_t T = a->seq_len;
    const bool qjl = a->key_format == KVQ_KEYS_QJL;
    // INT8: three 64 KB-ring CTAs per SM, about four waves of them; QJL: one 512-thread
    // CTA per SM (its byte tables fill shared memory), about two waves.
    const int64_t step = qjl ? kQjlTokPerStep : kInt8TokPerStep;
    const int64_t target = qjl ? (int64_t)sm_count * 2 : (int64_t)sm_count * 12;
    int64_t splits = pl.units > 0 ? (target + pl.units / 2) / pl.units : 1;
    const int64_t max_splits = (T + step - 1) / step;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    int64_t chunk = (T + splits - 1) / splits;
    chunk = (chunk + step - 1) / step * step;
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
        e = run_partial(true, G, p, pl.units, st);
    } else {
        e = run_partial(false, G, p, pl.units, st);
    }
    if (e != cudaSuccess || !a->out) return e;
    decode_combine_kernel<<<(unsigned)(a->batch * a->n_q_heads), kD, 0, st>>>(
        p.ws_ml, p.ws_acc, p.Hq, p.Hkv, pl.splits, a->out);
    return cudaGetLastError();
}

}  // namespace kvq
