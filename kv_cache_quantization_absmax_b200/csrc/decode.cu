// One decode step over a compressed KV cache: scores -> softmax -> weighted sum of
// INT8 values, for one query token per query head.
//
// Definitions: "GPU-Accelerated INT8 Quantization for KV Cache Compression in Large
// Language Models", abstract (attention scores over the INT8 cache); "QJL: 1-Bit
// Quantized JL Transform for KV Cache Quantization with Zero Overhead", abstract (the
// asymmetric estimator: the query's unquantized JL sketch against the key's sign bits);
// "Q-TensorFormer" model card, section 4 (GQA: query head h reads KV head h / G).
//
// Parallelisation (ours; the pages do not say how decode is parallelised).  The cached
// tokens of all (batch, KV head) units form one index space of units * T tokens, unit
// after unit, exactly as they lie in memory.  It is cut into equal contiguous ranges
// of W tokens (a multiple of 64), one per CTA, with as many CTAs as can be resident at
// once: every CTA streams its range exactly once with no refill gaps, and the load is
// balanced to within one stage whatever the number of units.  A range covers the end
// of one unit and the start of the next (or several short units): for each unit
// segment it touches, the CTA keeps an online-softmax state per query head of the
// group (running max m, running sum l, acc[D], base-2 domain) and writes it to slot
// (CTA, segment) of the workspace.  A second kernel merges, for every (batch, query
// head), the slots of the CTAs that covered its unit.  No kernel waits on another.
// Each K/V byte is read from HBM once and serves all G query heads of its group.
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "kvq_device.cuh"
#include "kvq_f32x2.cuh"
#include "kvq_int8.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kD = 128;
constexpr int kRange = 64;                 // CTA ranges are multiples of this many tokens
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kCodeMagic = 12583040.0f;  // 1.5 * 2^23 + 128
constexpr float kRoundMagic = 12582912.0f; // 1.5 * 2^23

struct DecodeParams {
    const uint16_t* q;
    const int8_t* kc;
    const float* ks;
    const uint32_t* kw;
    const uint16_t* kn;
    const int8_t* vc;
    const float* vs;
    float* sketch_v;        // QJL: the query projections [B * Hq][m] fp32 that a separate kernel
                            // writes; the tensor-core kernel's own slots [ctas][maxj - 1][G][256]
    float* scores_out;
    float* ws;              // partial states [ctas][maxj][G][2 + D]
    int64_t T;              // tokens attended per unit
    int64_t cap;            // cache rows per unit (row of token t of unit u: u * cap + t)
    const uint16_t* knew;   // append: new key rows [units][D] fp16, stored at token T - 1
    const uint16_t* vnew;   // append: new value rows [units][D] fp16 (or null)
    const uint16_t* S;      // append with QJL keys: the sketch matrix [m][D] fp16
    const uint8_t* v4p;     // INT4 values: packed codes [units * cap][D / 2]
    const float* v4s;       // INT4 values: group scales [units * cap][D / v4g]
    const float* v4z;       // INT4 values: group zero points
    int v4g;                // INT4 values: group size (32, 64 or 128)
    int v4_bulk;            // INT4 values: groups of 32 with 16-byte aligned parameters ->
                            // their scales and zero points are staged with the rows
    const uint8_t* k4p;     // residual keys: INT4 codes [units * cap][D / 2]
    const float* k4s;       // residual keys: group scales [units * cap][D / k4g]
    const float* k4z;       // residual keys: group zero points
    int k4_ng_shift;        // residual keys: log2(D / k4g)
    int k4_g_shift;         // residual keys: log2(k4g)
    int64_t W;              // tokens per CTA range
    int64_t total;          // units * T
    int Hq;
    int Hkv;
    int Gt;                 // query heads per KV head (Hq / Hkv)
    int nsub;               // head subgroups per KV head: the kernel's G heads each; CTA c
                            // covers token range c / nsub for heads of subgroup c % nsub
    int maxj;               // unit segments a range can touch
    int m;
    float scale_log2;       // sm_scale * log2(e)
    float qjl_c;            // sqrt(pi/2) / m
    int want_out;
    int scales_bulk;        // INT8: scales 16-byte aligned per stage -> bulk-copied too
    int qjl_bulk;           // QJL: value rows 16-byte aligned -> each warp's next 32 value
                            // rows come by one bulk copy
    int cuda_cores;         // the caller asked for no tensor-core value pass
    int test_expire;        // testing the failure path: the tensor-core kernels issue no key loads
};

// The unit segments of CTA `cta`'s range: unit u, tokens [t0, t1) of that unit, slot j.
struct Segment {
    int64_t u, t0, t1;
    int j;
};
struct RangeWalk {
    int64_t r_begin, r_end, u_first, T;
    __device__ RangeWalk(const DecodeParams& p, int cta)
        : r_begin((int64_t)cta * p.W), r_end(min(p.total, (int64_t)cta * p.W + p.W)),
          u_first(((int64_t)cta * p.W) / p.T), T(p.T) {}
    __device__ int count() const { return (int)((r_end - 1) / T - u_first + 1); }
    __device__ Segment seg(int j) const {
        const int64_t u = u_first + j;
        Segment s;
        s.u = u;
        s.t0 = max(r_begin, u * T) - u * T;
        s.t1 = min(r_end, (u + 1) * T) - u * T;
        s.j = j;
        return s;
    }
};

using x2::add2;
using x2::fma2;
using x2::mul2;
using x2::pack2;
using x2::unpack2;

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

// 2^x with the hardware approximation (relative error about 2^-22; 2^-inf = 0), for
// the softmax weights and rescale factors in the token loops.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- append of a new token (kvq_decode_append) ----
// One warp quantizes one fp16 row of D = 128 values (lane l: values 4 l .. 4 l + 3) with
// the per-row absmax INT8 rule of kvq_quantize_int8, bit for bit (kvq_int8.cuh), and
// stores the 128 codes and the scale.
__device__ __forceinline__ void append_int8_row(const uint16_t* src, int8_t* codes, float* scale, int lane) {
    const uint2 raw = *reinterpret_cast<const uint2*>(src + 4 * lane);
    const __half2* h = reinterpret_cast<const __half2*>(&raw);
    const float2 x01 = __half22float2(h[0]), x23 = __half22float2(h[1]);
    const float f[4] = {x01.x, x01.y, x23.x, x23.y};
    const float a_lane = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
    // max of non-negative floats = max of their bit patterns as unsigned integers
    const float a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a_lane)));
    const float sc = i8::row_scale(a);
    uint32_t word;
    i8::quantize_values<4>(f, sc, i8::scale_reciprocal(sc), &word);
    *reinterpret_cast<uint32_t*>(codes + 4 * lane) = word;
    if (lane == 0) *scale = sc;
}

// One warp writes sign word `w` (sketch rows 32 w .. 32 w + 31) of a new key: lane l
// computes (S k)_{32 w + l} in fp32 from the fp16 S row and key.
__device__ __forceinline__ uint32_t append_sign_word(const uint16_t* S, const uint16_t* k, int w, int lane) {
    const uint4* srow = reinterpret_cast<const uint4*>(S + (int64_t)(32 * w + lane) * kD);
    const uint4* kv = reinterpret_cast<const uint4*>(k);
    float acc = 0.0f;
#pragma unroll 4
    for (int c = 0; c < kD / 8; ++c) {
        const uint4 sv = __ldg(srow + c);
        const uint4 kk = __ldg(kv + c);  // the same 16 bytes in every lane
        const __half2* sh = reinterpret_cast<const __half2*>(&sv);
        const __half2* kh = reinterpret_cast<const __half2*>(&kk);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 a = __half22float2(sh[i]), b = __half22float2(kh[i]);
            acc = __fmaf_rn(a.x, b.x, acc);
            acc = __fmaf_rn(a.y, b.y, acc);
        }
    }
    return __ballot_sync(0xffffffffu, acc >= 0.0f);
}

// fp16 bits of ||k|| by the defining sequence: squares summed in fp64 in index order,
// IEEE square root, one rounding to fp16 (one thread).
__device__ __forceinline__ uint16_t append_norm_bits(const uint16_t* k) {
    double s64 = 0.0;
#pragma unroll 1
    for (int j = 0; j < kD; ++j) {
        const double d = (double)__half2float(__ushort_as_half(k[j]));
        s64 = __fma_rn(d, d, s64);
    }
    return __half_as_ushort(__double2half(__dsqrt_rn(s64)));
}

// The append of every unit's new token as a kernel of its own, for decodes that then run
// a tensor-core kernel (which does not encode it): one CTA per unit stores row T - 1.
// INT8 keys: warp 0 the key row, warp 1 the value row.  QJL keys: warps 0 .. m/32 - 1 one
// sign word each, warp m/32 the norm, warp m/32 + 1 the value row.  The rows are the same
// bits as the encode kernels' (and as the decode kernels' own append prologues).
__global__ void __launch_bounds__(32 * 10)
append_encode_kernel(const DecodeParams p, int qjl) {
    const int64_t u = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row = u * p.cap + p.T - 1;
    const uint16_t* kn = p.knew + u * kD;
    const int nw = qjl ? p.m / 32 : 1;
    if (qjl && warp < nw) {
        const uint32_t word = append_sign_word(p.S, kn, warp, lane);
        if (lane == 0) const_cast<uint32_t*>(p.kw)[row * nw + warp] = word;
    } else if (qjl && warp == nw) {
        if (lane == 0) const_cast<uint16_t*>(p.kn)[row] = append_norm_bits(kn);
    } else if (!qjl && warp == 0) {
        append_int8_row(kn, const_cast<int8_t*>(p.kc) + row * kD, const_cast<float*>(p.ks) + row, lane);
    } else if (warp == nw + (qjl ? 1 : 0) && p.vnew != nullptr) {
        append_int8_row(p.vnew + u * kD, const_cast<int8_t*>(p.vc) + row * kD, const_cast<float*>(p.vs) + row, lane);
    }
}

// Merge of per-warp softmax states (m, l, acc[D]) through shared memory into the
// segment's partial slot.  red: [WARPS][G][2 + kD] floats, already written.
template <int G, int WARPS>
__device__ __forceinline__ void merge_warps_and_store(const float* red, const DecodeParams& p,
                                                      int cta, int j, int tid, int nthreads) {
    for (int idx = tid; idx < G * kD; idx += nthreads) {
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
        float* slot = p.ws + (((int64_t)cta * p.maxj + j) * G + g) * (2 + kD);
        slot[2 + d] = a;
        if (d == 0) {
            slot[0] = mx;
            slot[1] = l;
        }
    }
}

// -----------------------------------------------------------------------------------
// INT8 keys.  The CTA's range streams through a shared-memory ring of stages of up to
// 64 or 128 tokens of one unit (K rows, V rows, and the scales when they are 16-byte
// aligned) filled by bulk asynchronous copies that one producer thread issues; eight
// consumer warps read the stage from shared memory.  LPT lanes share a token (8 lanes of
// 16 dims for up to two query heads per KV head, 16 lanes of 8 dims for four or eight;
// lane `sub` owns dims DPL sub .. DPL sub + DPL - 1 of K and V); each lane group takes U
// consecutive tokens of a stage and keeps its own online-softmax state; at the end of each unit
// segment the states are merged across groups (shuffles) and warps (shared memory)
// into the segment's slot while the producer already streams the next segment.
// -----------------------------------------------------------------------------------
// Ring geometry per group size G (measured on B200: for G = 1, two 128-token stages
// with three CTAs per SM beat four 64-token stages, the per-stage bookkeeping being
// spread over 4 tokens per lane group instead of 2).
template <int G, bool V4 = false>
struct I8Ring {
    static constexpr int tok = G == 1 ? 128 : 64;             // tokens per stage
    static constexpr int stages = G == 1 ? 2 : 4;
    static constexpr int vrow = V4 ? kD / 2 : kD;             // bytes of a value row
    // K rows | V rows | K scales | V scales | (INT4 values in groups of 32: the 4 group
    // scales, then the 4 zero points of each token)
    static constexpr int v_off = tok * kD;
    static constexpr int ks_off = v_off + tok * vrow;
    static constexpr int vs_off = ks_off + tok * 4;
    static constexpr int s4_off = vs_off + tok * 4;
    static constexpr int z4_off = s4_off + (V4 ? tok * 16 : 0);
    static constexpr int bytes = z4_off + (V4 ? tok * 16 : 0);
};
constexpr int kI8Consumers = 8;                          // consumer warps; warp 8 produces
constexpr int kI8Threads = 32 * (kI8Consumers + 1);

__device__ unsigned int g_decode_error = 0;

enum : unsigned int { kErrI8Producer = 0x201, kErrI8Consumer = 0x202, kErrQjlStep = 0x203 };

// Resident INT8 CTAs per SM the register budget is shaped for (more heads per group
// need more registers per thread).
__host__ __device__ constexpr int int8_ctas_per_sm(int G) { return G == 1 ? 3 : (G == 2 ? 2 : 1); }

// The byte tables of the sign-sketch estimator (the layout of the QJL decode kernel's
// tables, described there): entry (pos, b) holds, for each of the G
// heads, sum_{k<8} v[8 pos + k] * (bit k of b ? +1 : -1), at byte offset
// (pos / 16) * 64 KB + b * 256 + (pos % 16) * 16.
//
// The 16 entries (pos, b) with high nibble c of b, from the eight projections vv[g][k] =
// v[8 pos + k] of each head: the low nibble walks a Gray code, one sign flip per entry.
template <int G>
__device__ __forceinline__ void write_sign_entries(float* lut, int pos, int c, const float (&vv)[G][8]) {
    constexpr int HALF_FLOATS = 256 * 16 * 4;
    float val[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float sacc = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) sacc -= vv[g][k];
#pragma unroll
        for (int k = 0; k < 4; ++k) sacc += ((c >> k) & 1) ? vv[g][4 + k] : -vv[g][4 + k];
        val[g] = sacc;
    }
    float* base = lut + (pos >> 4) * HALF_FLOATS + (c * 16 * 16 + (pos & 15)) * 4;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int gray = i ^ (i >> 1);
        if (i > 0) {
            const int k = (i & 1) ? 0 : ((i & 2) ? 1 : ((i & 4) ? 2 : 3));   // the bit that flips at step i
            const bool on = (gray >> k) & 1;
#pragma unroll
            for (int g = 0; g < G; ++g) val[g] += on ? 2.0f * vv[g][k] : -2.0f * vv[g][k];
        }
        *reinterpret_cast<float4*>(base + gray * 16 * 4) =
            make_float4(val[0], G > 1 ? val[G > 1 ? 1 : 0] : 0.0f, G > 2 ? val[G > 2 ? 2 : 0] : 0.0f,
                        G > 3 ? val[G > 3 ? 3 : 0] : 0.0f);
    }
}

// All the tables, from the projections v (fp32, head g at v + g * vstride), by `nthr` threads.
template <int G>
__device__ __forceinline__ void build_sign_tables(float* lut, const float* v, int m, int64_t vstride, int tid,
                                                  int nthr) {
    const int npos = m / 8;
    for (int item = tid; item < 512; item += nthr) {
        const int pos = item & 31;
        const int c = item >> 5;                       // high nibble of the byte value
        float vv[G][8];
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < 8; ++k) vv[g][k] = pos < npos ? __ldg(v + g * vstride + pos * 8 + k) : 0.0f;
        write_sign_entries<G>(lut, pos, c, vv);
    }
}

// All the tables, by eight warps, from projections held one sketch row per thread: lane
// `lane` of warp w holds v[g][32 w + lane] in sv[g] and the warp writes the entries of
// positions 4 w .. 4 w + 3, whose eight rows each it holds, exchanged by shuffles (lane:
// position 4 w + lane / 8, high nibbles lane % 8 and lane % 8 + 8).
template <int G>
__device__ __forceinline__ void build_sign_tables_from_rows(float* lut, const float (&sv)[G], int w, int lane) {
    float vv[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int k = 0; k < 8; ++k) vv[g][k] = __shfl_sync(0xffffffffu, sv[g], (lane & ~7) + k);
    const int pos = 4 * w + (lane >> 3);
    write_sign_entries<G>(lut, pos, lane & 7, vv);
    write_sign_entries<G>(lut, pos, (lane & 7) + 8, vv);
}

// A lane's BYTES consecutive bytes of a shared-memory row (16, 8 or 4) as 32-bit words.
template <int BYTES>
__device__ __forceinline__ void load_row_words(const unsigned char* src, uint32_t* w) {
    if constexpr (BYTES == 16) {
        const uint4 v = *reinterpret_cast<const uint4*>(src);
        w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
    } else if constexpr (BYTES == 8) {
        const uint2 v = *reinterpret_cast<const uint2*>(src);
        w[0] = v.x, w[1] = v.y;
    } else {
        w[0] = *reinterpret_cast<const uint32_t*>(src);
    }
}

// Eight 4-bit codes (one word: element 2i in the low nibble of byte i) -> four exact
// float pairs (elements 2k, 2k + 1).
__device__ __forceinline__ void nibbles8(uint32_t w, uint64_t* c) {
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        c[k] = add2(pack2(__uint_as_float(__byte_perm(lo, 0x4B400000u, 0x7650u + k)),
                          __uint_as_float(__byte_perm(hi, 0x4B400000u, 0x7650u + k))),
                    pack2(-kRoundMagic, -kRoundMagic));
}

// A lane's view of the byte tables when it scores its own token: the 32 entries of a
// token are read at positions rotated by x = lane & 7 (both the 16-byte entry within
// an 8-entry group and the byte order within a word pair), so that the eight lanes of a
// shared-memory phase hit distinct banks.
struct LutLane {
    uint32_t off16[8];
    uint32_t sel[4];
    bool swap_words;
    __device__ explicit LutLane(int lane) {
        const int x = lane & 7;
        swap_words = (x & 4) != 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) off16[e] = (uint32_t)((e ^ x) * 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) sel[e] = 0x6504u | ((uint32_t)((e ^ x) & 3) << 4);
    }
};

// The estimator's table sum for one token: sc[g] = sum over the 32 byte positions of
// the token's sign words w[0..7] of entry (pos, byte) for head g (tables at shared
// address lut_s, the layout of build_sign_tables).
template <int G>
__device__ __forceinline__ void lut_token_sums(const uint32_t* w, uint32_t lut_s, const LutLane& L, float* sc) {
    constexpr int HALF_FLOATS = 256 * 16 * 4;
#pragma unroll
    for (int g = 0; g < G; ++g) sc[g] = 0.0f;
    uint64_t s01 = 0ull, s23 = 0ull, t01 = 0ull, t23 = 0ull;
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
        const uint32_t wa = L.swap_words ? w[2 * pr + 1] : w[2 * pr];
        const uint32_t wb = L.swap_words ? w[2 * pr] : w[2 * pr + 1];
        const uint32_t half_off = (uint32_t)((pr >> 1) * HALF_FLOATS * 4 + (pr & 1) * 128);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t o = __byte_perm(e < 4 ? wa : wb, L.off16[e], L.sel[e & 3]);
            const uint32_t addr = lut_s + half_off + o;
            if constexpr (G == 4) {
                float4 f;
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(f.x), "=f"(f.y), "=f"(f.z), "=f"(f.w) : "r"(addr));
                if (e & 1) {
                    t01 = add2(t01, pack2(f.x, f.y));
                    t23 = add2(t23, pack2(f.z, f.w));
                } else {
                    s01 = add2(s01, pack2(f.x, f.y));
                    s23 = add2(s23, pack2(f.z, f.w));
                }
            } else if constexpr (G == 2) {
                float2 f;
                asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(f.x), "=f"(f.y) : "r"(addr));
                if (e & 1) t01 = add2(t01, pack2(f.x, f.y));
                else s01 = add2(s01, pack2(f.x, f.y));
            } else {
                float f;
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f) : "r"(addr));
                sc[0] += f;
            }
        }
    }
    if constexpr (G >= 2) {
        const float2 a = unpack2(add2(s01, t01));
        sc[0] = a.x;
        sc[1] = a.y;
    }
    if constexpr (G == 4) {
        const float2 a = unpack2(add2(s23, t23));
        sc[2] = a.x;
        sc[3] = a.y;
    }
}

template <int G, bool V4>
__global__ void __launch_bounds__(kI8Threads, int8_ctas_per_sm(G))
decode_int8_kernel(const DecodeParams p) {
    using Ring = I8Ring<G, V4>;
    constexpr int kI8StageTok = Ring::tok;
    constexpr int kI8Stages = Ring::stages;
    constexpr int kI8StageBytes = Ring::bytes;
    // Lanes per token: 8 (16 dims each) up to two heads per KV head, 16 (8 dims each) for
    // more, which halves the per-lane query and accumulator state.
    constexpr int LPT = G >= 4 ? 16 : 8;
    constexpr int DPL = kD / LPT;          // dims per lane
    constexpr int NP = DPL / 2;            // packed fp32 pairs per lane
    constexpr int GPW = 32 / LPT;          // lane groups per warp
    static_assert(kI8StageTok % (GPW * kI8Consumers) == 0, "each lane group takes whole tokens");
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ uint64_t bars[2 * kI8Stages + 1];
    __shared__ int abort_storage;
    volatile int* abort_flag = &abort_storage;
    constexpr int U = kI8StageTok / (kI8Consumers * GPW);  // tokens per lane group per stage
    const int cta = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const RangeWalk walk(p, cta / p.nsub);
    const int nseg = walk.count();
    const uint32_t ring = dev::smem_u32(smem_raw);
    float* red = reinterpret_cast<float*>(smem_raw + kI8Stages * kI8StageBytes);  // [warps][G][2+D]
    const uint32_t bar0 = dev::smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (kI8Stages + s); };
    const uint32_t append_bar = bar0 + 8u * (2 * kI8Stages);  // appended rows are in global memory

    if (threadIdx.x == 0) {
        abort_storage = 0;
        for (int s = 0; s < kI8Stages; ++s) {
            dev::mbar_init(full_bar(s), 1);
            dev::mbar_init(empty_bar(s), kI8Consumers);
        }
        dev::mbar_init(append_bar, kI8Consumers);
        dev::mbar_init_fence();
    }
    __syncthreads();
    dev::griddep_launch_dependents();  // the combine kernel may be scheduled (it waits)

    if (warp == kI8Consumers) {
        // ---------------- producer ----------------
        if (lane == 0) {
            bool issued[kI8Stages];
            uint32_t ph_issued[kI8Stages];
            for (int s = 0; s < kI8Stages; ++s) issued[s] = false, ph_issued[s] = 0;
            int i = 0;
            bool run = true;
            bool appended_visible = false;
            for (int jj = 0; run && jj < nseg; ++jj) {
                const Segment sg = walk.seg(jj);
                const int64_t row0 = sg.u * p.cap;
                for (int64_t t = sg.t0; t < sg.t1; t += kI8StageTok, ++i) {
                    const int s = i % kI8Stages;
                    const uint32_t ph = (uint32_t)(i / kI8Stages) & 1u;
                    if (!dev::mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, &g_decode_error, kErrI8Producer)) {
                        run = false;
                        break;
                    }
                    const uint32_t n = (uint32_t)min((int64_t)kI8StageTok, sg.t1 - t);
                    if (p.knew != nullptr && !appended_visible && sg.t1 == p.T && t + n == sg.t1) {
                        // this stage holds a token the consumers append: copy it only once
                        // they have stored it (and made it visible to the async proxy)
                        if (!dev::mbar_wait(append_bar, 0u, abort_flag, &g_decode_error, kErrI8Producer)) {
                            run = false;
                            break;
                        }
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        appended_visible = true;
                    }
                    const uint32_t dst = ring + (uint32_t)s * kI8StageBytes;
                    // Values are copied only when the output is wanted (scores-only calls
                    // pass no value pointers); scales only when their rows start 16-byte
                    // aligned.
                    // (INT4 values: packed rows here, group scales and zero points loaded by
                    // the consumers)
                    const bool g32 = V4 && p.v4_bulk && p.want_out;  // group params staged too
                    const uint32_t k_bytes = n * kD + (p.scales_bulk ? n * 4u : 0u);
                    const uint32_t v_bytes = !p.want_out ? 0u
                                             : n * Ring::vrow + ((!V4 && p.scales_bulk) ? n * 4u : 0u) +
                                                   (g32 ? 2u * n * 16u : 0u);
                    dev::mbar_arrive_expect_tx(full_bar(s), k_bytes + v_bytes);
                    dev::bulk_g2s(dst, p.kc + (row0 + t) * kD, n * kD, full_bar(s));
                    if (p.want_out) {
                        if (g32) {
                            dev::bulk_g2s(dst + Ring::s4_off, p.v4s + (row0 + t) * 4, n * 16u, full_bar(s));
                            dev::bulk_g2s(dst + Ring::z4_off, p.v4z + (row0 + t) * 4, n * 16u, full_bar(s));
                        }
                        if constexpr (V4)
                            dev::bulk_g2s(dst + Ring::v_off, p.v4p + (row0 + t) * Ring::vrow, n * Ring::vrow,
                                          full_bar(s));
                        else
                            dev::bulk_g2s(dst + Ring::v_off, p.vc + (row0 + t) * kD, n * kD, full_bar(s));
                    }
                    if (p.scales_bulk) {
                        dev::bulk_g2s(dst + Ring::ks_off, p.ks + row0 + t, n * 4u, full_bar(s));
                        if (!V4 && p.want_out)
                            dev::bulk_g2s(dst + Ring::vs_off, p.vs + row0 + t, n * 4u, full_bar(s));
                    }
                    issued[s] = true;
                    ph_issued[s] = ph;
                }
            }
            for (int s = 0; s < kI8Stages; ++s)
                if (issued[s]) dev::mbar_drain(full_bar(s), ph_issued[s]);
        }
        __syncwarp();
        __syncthreads();  // matches the consumers' final barrier
        return;
    }

    // ---------------- consumers (warps 0 .. kI8Consumers-1) ----------------
    if (p.knew != nullptr) {
        // Append: the new token of every unit whose last token lies in this range is
        // quantized here (one warp per unit and row) and stored at token T - 1 before the
        // producer copies the stage holding it.
        int k = 0;
        for (int jj = 0; jj < nseg; ++jj) {
            const Segment sg = walk.seg(jj);
            if (sg.t1 != p.T) continue;
            if ((k++ % kI8Consumers) != warp) continue;
            const int64_t row = sg.u * p.cap + p.T - 1;
            append_int8_row(p.knew + sg.u * kD, const_cast<int8_t*>(p.kc) + row * kD,
                            const_cast<float*>(p.ks) + row, lane);
            if (p.vnew != nullptr)
                append_int8_row(p.vnew + sg.u * kD, const_cast<int8_t*>(p.vc) + row * kD,
                                const_cast<float*>(p.vs) + row, lane);
        }
        // visible to the producer's bulk copies (async proxy) and, through the barrier
        // below, to the other consumer warps' direct scale loads
        __threadfence();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(append_bar);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kI8Consumers) : "memory");
    }
    const int tg = lane / LPT;
    const int sub = lane % LPT;
    int i = 0;
    bool aborted = false;
    for (int jj = 0; jj < nseg; ++jj) {
        const Segment sg = walk.seg(jj);
        const int64_t row0 = sg.u * p.cap;
        const int64_t b = sg.u / p.Hkv;
        const int kvh = (int)(sg.u % p.Hkv);
        const int64_t hb = b * p.Hq + (int64_t)kvh * p.Gt + (int64_t)(cta % p.nsub) * G;
        uint64_t qp[G][NP];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const uint4* src = reinterpret_cast<const uint4*>(p.q + (hb + g) * kD + sub * DPL);
#pragma unroll
            for (int v = 0; v < DPL / 8; ++v) {
                const uint4 a = __ldg(src + v);
                const __half2* ha = reinterpret_cast<const __half2*>(&a);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f0 = __half22float2(ha[k]);
                    qp[g][4 * v + k] = pack2(f0.x, f0.y);
                }
            }
        }
        float mrun[G], lrun[G];
        uint64_t acc[G][NP];
        float zacc[G];  // INT4 values: sum over tokens of p * zero point (the same for the lane's dims)
#pragma unroll
        for (int g = 0; g < G; ++g) {
            mrun[g] = -INFINITY;
            lrun[g] = 0.0f;
            zacc[g] = 0.0f;
#pragma unroll
            for (int k = 0; k < NP; ++k) acc[g][k] = 0ull;
        }

        for (int64_t tstage = sg.t0; tstage < sg.t1; tstage += kI8StageTok, ++i) {
            const int s = i % kI8Stages;
            const uint32_t ph = (uint32_t)(i / kI8Stages) & 1u;
            const int tok0 = warp * (GPW * U) + tg * U;      // first token of this group in the stage
            const int rem = (int)min((int64_t)kI8StageTok, sg.t1 - tstage);  // tokens of the stage in range
            bool valid[U];
            float ksc[U], vsc[U], vz[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                valid[u] = tok0 + u < rem;
                const int64_t r = row0 + tstage + (valid[u] ? tok0 + u : 0);
                if (!p.scales_bulk) {
                    // coherent loads: an appended row's scales were stored by this kernel
                    ksc[u] = __ldcg(p.ks + r);
                    if constexpr (!V4) vsc[u] = p.want_out ? __ldcg(p.vs + r) : 0.0f;
                }
                if constexpr (V4) {
                    // this lane's dims lie in one group (groups of 32, 64 or 128); groups
                    // of 32 come with the stage, the others are loaded here
                    if (!p.v4_bulk && p.want_out) {
                        const int ng = kD / p.v4g;
                        const int64_t gi = r * ng + (sub * DPL) / p.v4g;
                        vsc[u] = __ldcg(p.v4s + gi);
                        vz[u] = __ldcg(p.v4z + gi);
                    } else {
                        vsc[u] = 0.0f;
                        vz[u] = 0.0f;
                    }
                } else {
                    vz[u] = 0.0f;
                }
            }
            // After an abort a warp keeps walking the same stages and barriers (so every
            // named barrier below still sees all consumer warps) but waits and computes
            // nothing more.
            if (!aborted) {
                const bool ok = dev::mbar_wait(full_bar(s), ph, abort_flag, &g_decode_error, kErrI8Consumer);
                aborted = !__all_sync(0xffffffffu, ok);
            }
            if (aborted) continue;
            const unsigned char* kst = smem_raw + (size_t)s * kI8StageBytes;
            const unsigned char* vst = kst + Ring::v_off;
            if constexpr (V4) {
                if (p.v4_bulk && p.want_out) {
                    const float* s4s = reinterpret_cast<const float*>(kst + Ring::s4_off);
                    const float* z4s = reinterpret_cast<const float*>(kst + Ring::z4_off);
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        vsc[u] = s4s[(tok0 + u) * 4 + ((sub * DPL) >> 5)];
                        vz[u] = z4s[(tok0 + u) * 4 + ((sub * DPL) >> 5)];
                    }
                }
            }
            if (p.scales_bulk) {
                // the group's U consecutive scales in one 8- or 16-byte load (tok0 is a
                // multiple of U and the scale arrays start 16-byte aligned in the stage)
                const float* kss = reinterpret_cast<const float*>(kst + Ring::ks_off) + tok0;
                const float* vss = reinterpret_cast<const float*>(kst + Ring::vs_off) + tok0;
                if constexpr (U == 4) {
                    const float4 k4 = *reinterpret_cast<const float4*>(kss);
                    ksc[0] = k4.x, ksc[1] = k4.y, ksc[2] = k4.z, ksc[3] = k4.w;
                    if constexpr (!V4) {
                        const float4 v4 = p.want_out ? *reinterpret_cast<const float4*>(vss) : make_float4(0, 0, 0, 0);
                        vsc[0] = v4.x, vsc[1] = v4.y, vsc[2] = v4.z, vsc[3] = v4.w;
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < U; u += 2) {
                        const float2 k2 = *reinterpret_cast<const float2*>(kss + u);
                        ksc[u] = k2.x, ksc[u + 1] = k2.y;
                        if constexpr (!V4) {
                            const float2 v2 = p.want_out ? *reinterpret_cast<const float2*>(vss + u) : make_float2(0, 0);
                            vsc[u] = v2.x, vsc[u + 1] = v2.y;
                        }
                    }
                }
            }
            float score[U][G];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                uint32_t w4[DPL / 4];
                load_row_words<DPL>(kst + (tok0 + u) * kD + sub * DPL, w4);
                uint64_t c[NP];
#pragma unroll
                for (int k = 0; k < DPL / 4; ++k) codes4(w4[k] ^ 0x80808080u, c[2 * k], c[2 * k + 1]);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    uint64_t dp0 = 0ull, dp1 = 0ull;
#pragma unroll
                    for (int k = 0; k < NP; k += 2) {
                        dp0 = fma2(qp[g][k], c[k], dp0);
                        dp1 = fma2(qp[g][k + 1], c[k + 1], dp1);
                    }
                    const float2 d2 = unpack2(add2(dp0, dp1));
                    float d = d2.x + d2.y;
#pragma unroll
                    for (int off = 1; off < LPT; off <<= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                    score[u][g] = d * ksc[u];
                }
            }
            if (p.scores_out != nullptr && sub == 0) {
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (valid[u]) {
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            p.scores_out[(hb + g) * p.T + tstage + tok0 + u] =
                                score[u][g];
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
                        const float corr = fast_exp2(mrun[g] - mb);
                        lrun[g] *= corr;
                        if constexpr (V4) zacc[g] *= corr;
                        const uint64_t c2 = pack2(corr, corr);
#pragma unroll
                        for (int k = 0; k < NP; ++k) acc[g][k] = mul2(acc[g][k], c2);
                        mrun[g] = mb;
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (!valid[u]) continue;
                    uint64_t c[NP];
                    if constexpr (V4) {
                        // DPL nibbles: byte i holds dims 2i (low) and 2i + 1 (high) -> the pairs
                        uint32_t wds[DPL / 8];
                        load_row_words<DPL / 2>(vst + (tok0 + u) * Ring::vrow + sub * (DPL / 2), wds);
#pragma unroll
                        for (int h = 0; h < DPL / 8; ++h) nibbles8(wds[h], c + 4 * h);
                    } else {
                        uint32_t w4[DPL / 4];
                        load_row_words<DPL>(vst + (tok0 + u) * kD + sub * DPL, w4);
#pragma unroll
                        for (int k = 0; k < DPL / 4; ++k) codes4(w4[k] ^ 0x80808080u, c[2 * k], c[2 * k + 1]);
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float pe = fast_exp2(score[u][g] * p.scale_log2 - mrun[g]);
                        lrun[g] += pe;
                        const float wv = pe * vsc[u];
                        if constexpr (V4) zacc[g] = __fmaf_rn(pe, vz[u], zacc[g]);
                        const uint64_t w2 = pack2(wv, wv);
#pragma unroll
                        for (int k = 0; k < NP; ++k) acc[g][k] = fma2(w2, c[k], acc[g][k]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(empty_bar(s));
        }
        if (!p.want_out) continue;

        // ---- end of the unit segment: merge lane groups, then warps, into slot jj ----
        if constexpr (V4) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const uint64_t z2 = pack2(zacc[g], zacc[g]);
#pragma unroll
                for (int k = 0; k < NP; ++k) acc[g][k] = add2(acc[g][k], z2);
            }
        }
#pragma unroll
        for (int off = LPT; off <= 16; off <<= 1) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float mo = __shfl_xor_sync(0xffffffffu, mrun[g], off);
                const float lo = __shfl_xor_sync(0xffffffffu, lrun[g], off);
                const float mn = fmaxf(mrun[g], mo);
                const float f1 = mn == -INFINITY ? 0.0f : exp2f(mrun[g] - mn);
                const float f2 = mn == -INFINITY ? 0.0f : exp2f(mo - mn);
                lrun[g] = lrun[g] * f1 + lo * f2;
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    const float2 a = unpack2(acc[g][k]);
                    const float ax = __shfl_xor_sync(0xffffffffu, a.x, off);
                    const float ay = __shfl_xor_sync(0xffffffffu, a.y, off);
                    acc[g][k] = pack2(a.x * f1 + ax * f2, a.y * f1 + ay * f2);
                }
                mrun[g] = mn;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kI8Consumers) : "memory");  // red[] is free
        if (tg == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float* r = red + (warp * G + g) * (2 + kD);
                if (sub == 0) {
                    r[0] = mrun[g];
                    r[1] = lrun[g];
                }
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    const float2 a = unpack2(acc[g][k]);
                    r[2 + sub * DPL + 2 * k] = a.x;
                    r[2 + sub * DPL + 2 * k + 1] = a.y;
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kI8Consumers) : "memory");
        merge_warps_and_store<G, kI8Consumers>(red, p, cta, jj, threadIdx.x, 32 * kI8Consumers);
    }
    __syncthreads();  // matches the producer warp's final barrier
}

// -----------------------------------------------------------------------------------
// QJL keys.  For each unit segment of the CTA's range, a warp takes 32 tokens per step.
//  * Byte tables (rebuilt per unit): LUT[p][b] (G floats) = sum_{k<8} v_g[8p + k] *
//    (bit k of b ? +1 : -1), stored as two halves of 16 positions, entry (p, b) at
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
template <int G, int THREADS>
__global__ void __launch_bounds__(THREADS, 1)
decode_qjl_kernel(const DecodeParams p) {
    extern __shared__ float4 dsmem4[];
    float* dsmem = reinterpret_cast<float*>(dsmem4);
    static_assert(THREADS >= 512 && THREADS % 32 == 0, "the table build uses 512 threads");
    constexpr int WARPS = THREADS / 32;
    constexpr int TOK_PER_STEP = WARPS * 32;
    constexpr int HALF_FLOATS = 256 * 16 * 4;        // one table half: 64 KB
    const int cta = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const RangeWalk walk(p, cta / p.nsub);
    const int nseg = walk.count();
    const int nw = p.m / 32;
    const int npos = p.m / 8;
    float* lut = dsmem;                              // 2 halves x [256][16] x 4 floats
    float* wbuf = dsmem + 2 * HALF_FLOATS;           // [WARPS][16 pairs][G][2]
    float* red = dsmem;                              // [WARPS][G][2 + kD], reuses the tables

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
    dev::griddep_launch_dependents();  // the combine kernel may be scheduled (it waits)

    if (p.knew != nullptr) {
        // Append: the new token of every unit whose last token lies in this range is
        // encoded here (warps 0 .. m/32 - 1: one sign word each; warp m/32: the norm;
        // warp m/32 + 1: the INT8 value row) and stored at token T - 1; the barrier
        // below orders these stores before the loads of the segment loop.
        for (int jj = 0; jj < nseg; ++jj) {
            const Segment sg = walk.seg(jj);
            if (sg.t1 != p.T) continue;
            const int64_t row = sg.u * p.cap + p.T - 1;
            const uint16_t* kn = p.knew + sg.u * kD;
            if (warp < nw) {
                const uint32_t word = append_sign_word(p.S, kn, warp, lane);
                if (lane == 0) const_cast<uint32_t*>(p.kw)[row * nw + warp] = word;
            } else if (warp == nw) {
                if (lane == 0) const_cast<uint16_t*>(p.kn)[row] = append_norm_bits(kn);
            } else if (warp == nw + 1 && p.vnew != nullptr) {
                append_int8_row(p.vnew + sg.u * kD, const_cast<int8_t*>(p.vc) + row * kD,
                                const_cast<float*>(p.vs) + row, lane);
            }
        }
        __threadfence();
        __syncthreads();
    }
    float* mybuf = wbuf + warp * 32 * G;
    const uint64_t magic = pack2(-kCodeMagic, -kCodeMagic);

    for (int jj = 0; jj < nseg; ++jj) {
        const Segment sg = walk.seg(jj);
        const int64_t row0 = sg.u * p.cap;
        const int64_t b = sg.u / p.Hkv;
        const int kvh = (int)(sg.u % p.Hkv);
        const int64_t hb = b * p.Hq + (int64_t)kvh * p.Gt + (int64_t)(cta % p.nsub) * G;
        __syncthreads();  // the previous segment's merge no longer reads red[]
        // ---- byte tables ----
        if (threadIdx.x < 512) {
            const int pos = threadIdx.x & 31;
            const int c = threadIdx.x >> 5;               // high nibble of the byte value
            float v[G][8];
    #pragma unroll
            for (int g = 0; g < G; ++g) {
                const float* src = p.sketch_v + (hb + g) * p.m + pos * 8;
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

        float mrun[G], lsum[G];
        uint64_t acc[G][4];                               // (even, odd) token partial sums, 4 dims
#pragma unroll
        for (int g = 0; g < G; ++g) {
            mrun[g] = -INFINITY;
            lsum[g] = 0.0f;
#pragma unroll
            for (int d = 0; d < 4; ++d) acc[g][d] = 0ull;
        }

        for (int64_t t0 = sg.t0 + (int64_t)warp * 32; t0 < sg.t1; t0 += TOK_PER_STEP) {
            const int nvalid = (int)min((int64_t)32, sg.t1 - t0);
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
                for (int k = 0; k < 8; ++k) w[k] = k < nw ? __ldcs(p.kw + r * nw + k) : 0u;
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
            uint64_t s01 = 0ull, s23 = 0ull, t01 = 0ull, t23 = 0ull;
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
                        if (e & 1) {
                            t01 = add2(t01, pack2(f.x, f.y));
                            t23 = add2(t23, pack2(f.z, f.w));
                        } else {
                            s01 = add2(s01, pack2(f.x, f.y));
                            s23 = add2(s23, pack2(f.z, f.w));
                        }
                    } else if constexpr (G == 2) {
                        float2 f;
                        asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(f.x), "=f"(f.y) : "r"(addr));
                        if (e & 1) t01 = add2(t01, pack2(f.x, f.y));
                        else s01 = add2(s01, pack2(f.x, f.y));
                    } else {
                        float f;
                        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(f) : "r"(addr));
                        sc[0] += f;
                    }
                }
            }
            if constexpr (G >= 2) {
                const float2 a = unpack2(add2(s01, t01));
                sc[0] = a.x;
                sc[1] = a.y;
            }
            if constexpr (G == 4) {
                const float2 a = unpack2(add2(s23, t23));
                sc[2] = a.x;
                sc[3] = a.y;
            }
            float score[G];
#pragma unroll
            for (int g = 0; g < G; ++g) score[g] = p.qjl_c * nrm * sc[g];
            if (p.scores_out != nullptr && valid) {
#pragma unroll
                for (int g = 0; g < G; ++g)
                    p.scores_out[(hb + g) * p.T + t0 + lane] = score[g];
            }
            if (!p.want_out) continue;
            // ---- online softmax at warp granularity ----
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float lg = valid ? score[g] * p.scale_log2 : -INFINITY;
                const float mb = warp_max(lg);
                if (mb > mrun[g]) {
                    const float corr = fast_exp2(mrun[g] - mb);
                    lsum[g] *= corr;
                    const uint64_t c2 = pack2(corr, corr);
#pragma unroll
                    for (int d = 0; d < 4; ++d) acc[g][d] = mul2(acc[g][d], c2);
                    mrun[g] = mb;
                }
                const float pe = fast_exp2(lg - mrun[g]);
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
        if (!p.want_out) continue;

        // ---- end of the unit segment: per-warp state -> shared memory -> slot jj ----
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], off);
        __syncthreads();  // the byte tables are no longer read
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
        merge_warps_and_store<G, WARPS>(red, p, cta, jj, threadIdx.x, THREADS);
    }
}


// -----------------------------------------------------------------------------------
// QJL keys, prefetching variant (16 warps, one CTA per SM).  The byte tables, the
// estimator lookups, the warp-level online softmax and the value pass are those of
// decode_qjl_kernel above; the difference is when a step's data is requested.  Each warp
// has the next step's sign words, norm and value scale loaded into registers while it
// computes the current step, and a 4 KB value buffer in shared memory that its lane 0
// refills with one bulk asynchronous copy (32 value rows) as soon as the value pass has
// read it, so the copy overlaps the next step's lookups and softmax (the wait on the
// buffer's mbarrier is bounded).  A step of fewer than 32 tokens (a range's tail) is
// staged into the buffer with ordinary loads.  The value codes no longer sit in 32
// registers per lane.
// -----------------------------------------------------------------------------------
constexpr int kQpfWarps = 16;
constexpr int kQpfThreads = 32 * kQpfWarps;
constexpr int kQpfSlot = 32 * kD;                       // 32 value rows

// RES: keys stored as group-wise INT4 plus the residual's sign sketch.  The lane of a
// token then also forms <q, k_hat> = sum_g s_g <q, c>_g + z_g sum_g q for its G heads
// from its 64 code bytes (direct loads) and the unit's queries, which sit in shared
// memory as fp32 and are read by broadcast; the sign words are the residual's and the
// estimator is scaled by the residual's norm.
template <int G, bool RES = false>
__global__ void __launch_bounds__(kQpfThreads, 1)
decode_qjl_pf_kernel(const DecodeParams p) {
    extern __shared__ float4 dsmem4[];
    float* dsmem = reinterpret_cast<float*>(dsmem4);
    constexpr int WARPS = kQpfWarps;
    constexpr int TOK_PER_STEP = WARPS * 32;
    constexpr int HALF_FLOATS = 256 * 16 * 4;        // one table half: 64 KB
    __shared__ uint64_t bars[WARPS];
    __shared__ int abort_storage;
    volatile int* abort_flag = &abort_storage;
    const int cta = blockIdx.x;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const RangeWalk walk(p, cta / p.nsub);
    const int nseg = walk.count();
    const int nw = p.m / 32;
    float* lut = dsmem;                              // 2 halves x [256][16] x 4 floats
    float* wbuf = dsmem + 2 * HALF_FLOATS;           // [WARPS][16 pairs][G][2]
    float* red = dsmem;                              // [WARPS][G][2 + kD], reuses the tables
    unsigned char* vbuf = reinterpret_cast<unsigned char*>(wbuf + WARPS * 32 * G) + (size_t)warp * kQpfSlot;
    // residual keys: the unit's queries [G][D] fp32 and their group sums [G][4]
    float* qs = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(wbuf + WARPS * 32 * G) +
                                         (size_t)WARPS * kQpfSlot);
    float* qgs = qs + G * kD;
    const uint32_t bar = dev::smem_u32(bars) + 8u * warp;

    const LutLane lut_lane(lane);
    const uint32_t lut_s = (uint32_t)__cvta_generic_to_shared(lut);

    if (threadIdx.x == 0) {
        abort_storage = 0;
        for (int b2 = 0; b2 < WARPS; ++b2) dev::mbar_init(dev::smem_u32(bars) + 8u * b2, 1);
        dev::mbar_init_fence();
    }
    __syncthreads();
    dev::griddep_launch_dependents();  // the combine kernel may be scheduled (it waits)

    float* mybuf = wbuf + warp * 32 * G;
    const uint64_t magic = pack2(-kCodeMagic, -kCodeMagic);
    int nissue = 0, ndone = 0;
    bool aborted = false;

    for (int jj = 0; jj < nseg; ++jj) {
        const Segment sg = walk.seg(jj);
        const int64_t row0 = sg.u * p.cap;
        const int64_t b = sg.u / p.Hkv;
        const int kvh = (int)(sg.u % p.Hkv);
        const int64_t hb = b * p.Hq + (int64_t)kvh * p.Gt + (int64_t)(cta % p.nsub) * G;
        __syncthreads();  // the previous segment's merge no longer reads red[]
        build_sign_tables<G>(lut, p.sketch_v + hb * p.m, p.m, p.m, threadIdx.x,
                             kQpfThreads);
        if constexpr (RES) {
            for (int i = threadIdx.x; i < G * kD; i += kQpfThreads)
                qs[i] = __half2float(__ushort_as_half(p.q[hb * kD + i]));
        }
        __syncthreads();
        if constexpr (RES) {
            const int ng = 1 << p.k4_ng_shift;
            if (threadIdx.x < G * ng) {
                const int g = threadIdx.x >> p.k4_ng_shift, gi = threadIdx.x & (ng - 1);
                const int len = 1 << p.k4_g_shift;
                float a = 0.0f;
                for (int j = 0; j < len; ++j) a += qs[g * kD + gi * len + j];
                qgs[g * 4 + gi] = a;
            }
            __syncthreads();
        }

        float mrun[G], lsum[G];
        uint64_t acc[G][4];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            mrun[g] = -INFINITY;
            lsum[g] = 0.0f;
#pragma unroll
            for (int d = 0; d < 4; ++d) acc[g][d] = 0ull;
        }
        // a whole block of 32 tokens: its value rows arrive by one bulk copy
        auto bulk_step = [&](int64_t t0) { return p.qjl_bulk && p.want_out && t0 + 32 <= sg.t1; };
        auto issue = [&](int64_t t0) {
            __syncwarp();   // every lane is done reading the buffer
            if (lane == 0) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                dev::mbar_arrive_expect_tx(bar, (uint32_t)kQpfSlot);
                dev::bulk_g2s(dev::smem_u32(vbuf), p.vc + (row0 + t0) * kD, (uint32_t)kQpfSlot, bar);
            }
            ++nissue;
        };
        // this lane's token of a step: sign words, norm, value scale (registers)
        auto load_small = [&](int64_t t0, uint32_t* w, float& nrm, float& vsc) {
            const bool v = t0 + lane < sg.t1;
            const int64_t r = row0 + t0 + (v ? lane : 0);
            if (nw == 8) {
                const uint4 a = __ldcs(reinterpret_cast<const uint4*>(p.kw + r * 8));
                const uint4 c = __ldcs(reinterpret_cast<const uint4*>(p.kw + r * 8) + 1);
                w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
                w[4] = c.x; w[5] = c.y; w[6] = c.z; w[7] = c.w;
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) w[k] = k < nw ? __ldcs(p.kw + r * nw + k) : 0u;
            }
            nrm = __half2float(__ushort_as_half(__ldcs(p.kn + r)));
            vsc = p.want_out ? __ldcs(p.vs + r) : 0.0f;
        };
        int64_t t0 = sg.t0 + (int64_t)warp * 32;
        uint32_t w[8];
        float nrm = 0.0f, vsc = 0.0f;
        if (t0 < sg.t1) {
            load_small(t0, w, nrm, vsc);
            if (!aborted && bulk_step(t0)) issue(t0);
        }
        for (; t0 < sg.t1; t0 += TOK_PER_STEP) {
            const int64_t tn = t0 + TOK_PER_STEP;
            uint32_t wn[8];
            float nrmn = 0.0f, vscn = 0.0f;
            if (tn < sg.t1) load_small(tn, wn, nrmn, vscn);     // the next step, in flight
            const int nvalid = (int)min((int64_t)32, sg.t1 - t0);
            const bool valid = lane < nvalid;
            if (!aborted) {
                // ---- estimator: 32 byte-table lookups ----
                float sc[G];
                lut_token_sums<G>(w, lut_s, lut_lane, sc);
                float score[G];
#pragma unroll
                for (int g = 0; g < G; ++g) score[g] = p.qjl_c * nrm * sc[g];
                if constexpr (RES) {
                    // ---- <q, k_hat> of this lane's token from its INT4 codes ----
                    const int64_t r = row0 + t0 + (valid ? lane : 0);
                    const uint4* crow = reinterpret_cast<const uint4*>(p.k4p + r * (kD / 2));
                    uint4 cw[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) cw[k] = __ldcs(crow + k);   // dims 32 k .. 32 k + 31
                    const int ng = 1 << p.k4_ng_shift;
                    const float* s4 = p.k4s + (r << p.k4_ng_shift);
                    const float* z4 = p.k4z + (r << p.k4_ng_shift);
                    float kdot[G];
#pragma unroll
                    for (int g = 0; g < G; ++g) kdot[g] = 0.0f;
                    // dims in blocks of 32 (one 16-byte code load); a block lies in one group
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int gi = (32 * k) >> p.k4_g_shift;
                        uint64_t part[G];
#pragma unroll
                        for (int g = 0; g < G; ++g) part[g] = 0ull;
                        const uint32_t wds[4] = {cw[k].x, cw[k].y, cw[k].z, cw[k].w};
#pragma unroll
                        for (int w8 = 0; w8 < 4; ++w8) {
                            uint64_t c[4];
                            nibbles8(wds[w8], c);
                            const int d0 = 32 * k + 8 * w8;
#pragma unroll
                            for (int g = 0; g < G; ++g) {
                                const float4 qa = *reinterpret_cast<const float4*>(qs + g * kD + d0);
                                const float4 qb = *reinterpret_cast<const float4*>(qs + g * kD + d0 + 4);
                                part[g] = fma2(pack2(qa.x, qa.y), c[0], part[g]);
                                part[g] = fma2(pack2(qa.z, qa.w), c[1], part[g]);
                                part[g] = fma2(pack2(qb.x, qb.y), c[2], part[g]);
                                part[g] = fma2(pack2(qb.z, qb.w), c[3], part[g]);
                            }
                        }
                        // the group's scale and zero point close each group of dims
                        const bool last = ((32 * (k + 1)) >> p.k4_g_shift) != gi || k == 3;
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float2 pp = unpack2(part[g]);
                            kdot[g] += pp.x + pp.y;
                        }
                        if (last) {
                            const float sg4 = __ldg(s4 + gi), zg4 = __ldg(z4 + gi);
#pragma unroll
                            for (int g = 0; g < G; ++g) {
                                score[g] = __fmaf_rn(kdot[g], sg4, __fmaf_rn(zg4, qgs[g * 4 + gi], score[g]));
                                kdot[g] = 0.0f;
                            }
                        }
                        (void)ng;
                    }
                }
                if (p.scores_out != nullptr && valid) {
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        p.scores_out[(hb + g) * p.T + t0 + lane] = score[g];
                }
                if (p.want_out) {
                    // ---- online softmax at warp granularity ----
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float lg = valid ? score[g] * p.scale_log2 : -INFINITY;
                        const float mb = warp_max(lg);
                        if (mb > mrun[g]) {
                            const float corr = fast_exp2(mrun[g] - mb);
                            lsum[g] *= corr;
                            const uint64_t c2 = pack2(corr, corr);
#pragma unroll
                            for (int d = 0; d < 4; ++d) acc[g][d] = mul2(acc[g][d], c2);
                            mrun[g] = mb;
                        }
                        const float pe = fast_exp2(lg - mrun[g]);
                        lsum[g] += pe;
                        mybuf[(lane >> 1) * (2 * G) + g * 2 + (lane & 1)] = pe * vsc;
                    }
                    // ---- this step's value rows ----
                    if (bulk_step(t0)) {
                        const bool ok = dev::mbar_wait(bar, (uint32_t)(ndone & 1), abort_flag, &g_decode_error,
                                                       kErrQjlStep);
                        aborted = !__all_sync(0xffffffffu, ok);
                        if (!aborted) ++ndone;
                    } else {
                        const unsigned int* vrow = reinterpret_cast<const unsigned int*>(p.vc + (row0 + t0) * kD) + lane;
                        for (int j = 0; j < 32; ++j)
                            reinterpret_cast<uint32_t*>(vbuf + j * kD)[lane] = j < nvalid ? __ldcs(vrow + j * (kD / 4))
                                                                                          : 0x80808080u;
                    }
                    __syncwarp();
                    if (!aborted) {
                        // ---- values: dims 4 lane .. 4 lane + 3, token pairs (2 jp, 2 jp + 1) ----
                        const uint32_t* vals = reinterpret_cast<const uint32_t*>(vbuf) + lane;
#pragma unroll
                        for (int jp = 0; jp < 16; ++jp) {
                            const uint32_t ce = vals[(2 * jp) * (kD / 4)] ^ 0x80808080u;
                            const uint32_t co = vals[(2 * jp + 1) * (kD / 4)] ^ 0x80808080u;
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
                        // the buffer is read: the next step's value rows may come in
                        if (tn < sg.t1 && bulk_step(tn)) issue(tn);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) w[k] = wn[k];
            nrm = nrmn;
            vsc = vscn;
        }
        if (!p.want_out) continue;

        // ---- end of the unit segment: per-warp state -> shared memory -> slot jj ----
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], off);
        __syncthreads();  // the byte tables are no longer read
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
        merge_warps_and_store<G, WARPS>(red, p, cta, jj, threadIdx.x, kQpfThreads);
    }
    // a copy still in flight after an abort completes before the CTA exits
    if (lane == 0 && nissue > ndone) dev::mbar_drain(bar, (uint32_t)((nissue - 1) & 1));
    __syncwarp();
}

// -----------------------------------------------------------------------------------
// QJL keys, value pass on the tensor cores.  The range streams in chunks of 128 tokens
// of one unit through two rings, each filled by its own producer thread: a key ring (the
// chunk's sign words, by bulk copies) and a value ring (the
// chunk's 128 value rows by a TMA tile with the 128-byte swizzle, which the tensor core
// reads as the MN-major operand A = V^T [128 dims x 128 tokens]).  A scorer takes a
// chunk's sign words as soon as they land and releases the key stage once it holds them
// in registers (the norms and value scales it loads itself), so a chunk's weights are
// usually ready before its value tile lands, and a value stage is held only for its load
// and its MMA.
// Warp roles (480 threads, one CTA per SM):
//   warp 0       key producer; warp 14 value producer;
//   warp 1       TMEM and the MMA thread: per chunk four tcgen05.mma kind::i8, slice k
//                (tokens 32 k .. 32 k + 31), all into the chunk's 16-column int32
//                accumulator;
//   warps 2..9   scorers, one warp per chunk (chunk c to warp c % 8), four tokens per
//                thread (tokens 32 i + lane, i = 0 .. 3, i.e. slice i): the estimator from
//                the byte tables; the chunk's max logit Mc of each head and max value scale
//                smax by warp reductions; the weight w = 2^(s - Mc) * vscale as a 24-bit
//                fixed-point integer W = round(w 2^E), 2^E the power of two that puts
//                smax 2^E in [2^23, 2^24), split into three unsigned bytes that form rows
//                3 g + k of the operand B [16 x 128 tokens] (K-major); the chunk's sum of
//                2^(s - Mc) in fixed point by one integer warp reduction per head;
//   warps 10..13 accumulators, one value dimension per thread: sum_t W_t c_t = D2 2^16 +
//                D1 2^8 + D0 (exact in int32: |c| <= 127, bytes <= 255, 128 tokens), times
//                2^-E, merged into the running online-softmax state of each head.
// The INT8 codes enter the product unconverted and every product and sum is exact; the
// approximations are the weights' fixed point (absolute error below 2^-23 smax per
// token: the product is rounded to fp32 before its rounding to the fixed point), the
// sums' 2^-24 fixed point (at most 2^-25 per token), and the fp32 merges.
constexpr int kTcTok = 128;                 // tokens per chunk
constexpr int kTcValueStages = 3;           // value ring: 16 KB tiles
constexpr int kTcScorerWarps = 8;           // one scorer warp per chunk, chunk c to warp c % 8
// Key stages: the sign words of a chunk, one stage per scorer warp (chunk c in stage c % 8),
// so that each stage has one consumer that takes its fills in order (mbarrier phases are
// told apart by parity only: a consumer must never be more than one fill ahead).
constexpr int kTcKeyStages = kTcScorerWarps;
static_assert(kTcScorerWarps == 8, "the scorers build the tables as eight warps of four positions");
// Units a CTA range may touch (the projections of all but the first wait in the workspace;
// shorter units go to the CUDA-core kernel)
constexpr int kTcMaxUnits = 9;
constexpr int kTcValueWarp = 2 + kTcScorerWarps + 4;   // the value producer, after the accumulators
constexpr int kTcThreads = 32 * (kTcValueWarp + 1);
constexpr int kTcVBytes = kTcTok * kD;      // value tile: 16 KB
constexpr int kTcKeyBytes = kTcTok * 32;    // key stage: the chunk's sign words (<= 4 KB)
constexpr int kTcBBytes = 2048;             // operand B: 16 rows x 128 bytes
constexpr int kTcAcc = kTcScorerWarps;       // chunks in flight between scorers and accumulators
constexpr uint32_t kTcTmemCols = kTcAcc * 16 <= 32 ? 32 : (kTcAcc * 16 <= 64 ? 64 : (kTcAcc * 16 <= 128 ? 128 : 256));
// instruction descriptor: int32 accumulator, A signed 8-bit MN-major, B unsigned 8-bit
// K-major, N = 16, M = 128
constexpr uint32_t kTcIdesc = (2u << 4) | (1u << 7) | (0u << 10) | (1u << 15) | (0u << 16) |
                              ((16u >> 3) << 17) | ((128u >> 4) << 24);

enum : unsigned int { kErrTcProducer = 0x211, kErrTcMma = 0x212, kErrTcScore = 0x213, kErrTcAcc = 0x214 };

struct TcChunk {              // per chunk in flight, from its scorer warp to the accumulators
    float Mc[4];              // [head] the chunk's max logit
    float L[4];               // [head] sum over the chunk of 2^(s - Mc)
    float inv;                // 2^-E: the value of one unit of the weights' fixed point
    float pad[3];
};

// Shared memory, from a 1024-byte aligned base: byte tables | value ring | operand B
// buffers | key ring | per-chunk statistics | mbarriers.
constexpr size_t kTcLutOff = 0;
constexpr size_t kTcValueOff = kTcLutOff + 2 * 65536;
constexpr size_t kTcBOff = kTcValueOff + (size_t)kTcValueStages * kTcVBytes;
constexpr size_t kTcKeyOff = kTcBOff + (size_t)kTcAcc * kTcBBytes;
constexpr size_t kTcSliceOff = kTcKeyOff + (size_t)kTcKeyStages * kTcKeyBytes;
constexpr size_t kTcBarOff = kTcSliceOff + (size_t)kTcAcc * sizeof(TcChunk);
constexpr int kTcBars = 2 * kTcKeyStages + 2 * kTcValueStages + 3 * kTcAcc + 2;
static_assert(kTcValueOff % 1024 == 0 && kTcBOff % 1024 == 0, "swizzled operands need 1024-byte alignment");
static_assert(kTcKeyBytes % 16 == 0 && kTcSliceOff % 16 == 0, "bulk copy destinations are 16-byte aligned");

__host__ __device__ constexpr size_t tc_smem_bytes() {
    return 1024 /* alignment */ + kTcBarOff + (size_t)kTcBars * 8;
}
static_assert(tc_smem_bytes() + 64 <= 232448, "shared memory of one CTA");

template <int G>
__global__ void __launch_bounds__(kTcThreads, 1)
decode_qjl_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap vmap) {
    extern __shared__ uint8_t tc_raw[];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_storage;
    volatile int* abort_flag = &abort_storage;
    const uint32_t raw = dev::smem_u32(tc_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* bp = tc_raw + (base - raw);
    float* lut = reinterpret_cast<float*>(bp + kTcLutOff);               // 128 KB
    const uint32_t lut_s = base + (uint32_t)kTcLutOff;
    const uint32_t val_s = base + (uint32_t)kTcValueOff;
    const uint32_t b_s = base + (uint32_t)kTcBOff;
    uint8_t* b_p = bp + kTcBOff;
    const uint32_t key_s = base + (uint32_t)kTcKeyOff;
    const uint8_t* key_p = bp + kTcKeyOff;
    TcChunk* chunks = reinterpret_cast<TcChunk*>(bp + kTcSliceOff);   // [kTcAcc]
    const uint32_t bars = base + (uint32_t)kTcBarOff;
    auto kfull_bar = [&](int s) { return bars + 8u * s; };
    auto kempty_bar = [&](int s) { return bars + 8u * (kTcKeyStages + s); };
    auto vfull_bar = [&](int s) { return bars + 8u * (2 * kTcKeyStages + s); };
    auto vempty_bar = [&](int s) { return bars + 8u * (2 * kTcKeyStages + kTcValueStages + s); };
    constexpr int kAccBar0 = 2 * kTcKeyStages + 2 * kTcValueStages;
    auto bready_bar = [&](int a) { return bars + 8u * (kAccBar0 + a); };
    auto tfull_bar = [&](int a) { return bars + 8u * (kAccBar0 + kTcAcc + a); };
    auto tempty_bar = [&](int a) { return bars + 8u * (kAccBar0 + 2 * kTcAcc + a); };
    const uint32_t done_bar = bars + 8u * (kAccBar0 + 3 * kTcAcc);
    const uint32_t pro_bar = bars + 8u * (kAccBar0 + 3 * kTcAcc + 1);   // the projection inputs

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const RangeWalk walk(p, cta / p.nsub);
    const int nseg = walk.count();
    const int nw = p.m / 32;
    // the first of the G query heads this CTA serves for unit u
    const auto tc_head0 = [&](int64_t u) {
        return (u / p.Hkv) * p.Hq + (u % p.Hkv) * p.Gt + (int64_t)(cta % p.nsub) * G;
    };

    if (threadIdx.x == 0) {
        abort_storage = 0;
        for (int s = 0; s < kTcKeyStages; ++s) {
            dev::mbar_init(kfull_bar(s), 1);
            dev::mbar_init(kempty_bar(s), 1);     // the chunk's scorer warp
        }
        for (int s = 0; s < kTcValueStages; ++s) {
            dev::mbar_init(vfull_bar(s), 1);
            dev::mbar_init(vempty_bar(s), 1);     // the MMA's commit
        }
        for (int a = 0; a < kTcAcc; ++a) {
            dev::mbar_init(bready_bar(a), 1);
            dev::mbar_init(tfull_bar(a), 1);
            dev::mbar_init(tempty_bar(a), 4);
        }
        dev::mbar_init(done_bar, 1);
        dev::mbar_init(pro_bar, 1);
        dev::mbar_init_fence();
    }
    // operand B: rows 3 G .. 15 stay zero
    for (int i = threadIdx.x; i < kTcAcc * kTcBBytes / 16; i += kTcThreads)
        reinterpret_cast<uint4*>(b_p)[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) dev::tmem_alloc(dev::smem_u32(&tmem_slot), kTcTmemCols);
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    dev::griddep_launch_dependents();  // the combine kernel may be scheduled (it waits)

    if (warp == 0 || warp == kTcValueWarp) {
        // ---------------- producers: warp 0 the key ring, warp kTcValueWarp the value ring ----------------
        // Two threads, so that a value tile is never held back behind a key load: at the
        // start of a new unit the scorers that have finished the old one wait for the
        // others at the table rebuild, and those may need the old unit's last value tiles.
        // (KVQ_DECODE_TEST_EXPIRE: the key producer issues nothing, its consumers' waits expire)
        if (lane == 0 && !(warp == 0 && p.test_expire)) {
            const bool keys = warp == 0;
            if (!keys)
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
            if (keys) {
                // the projection inputs, into the table space the scorers fill only after
                // they have used them: S (m rows of kD fp16) at 0 and the G query rows
                // of each unit this CTA visits after 64 KB
                dev::mbar_arrive_expect_tx(pro_bar, (uint32_t)(p.m * kD * 2 + nseg * G * kD * 2));
                dev::bulk_g2s(lut_s, p.S, (uint32_t)(p.m * kD * 2), pro_bar);
                for (int jj = 0; jj < nseg; ++jj)
                    dev::bulk_g2s(lut_s + 65536u + (uint32_t)(jj * G * kD * 2), p.q + tc_head0(walk.seg(jj).u) * kD,
                                  (uint32_t)(G * kD * 2), pro_bar);
            }
            int i = 0;
            bool ok = true;
            for (int jj = 0; ok && jj < nseg; ++jj) {
                const Segment sg = walk.seg(jj);
                for (int64_t t = sg.t0; t < sg.t1; t += kTcTok, ++i) {
                    const int64_t r = sg.u * p.cap + t;
                    if (keys) {
                        const int s = i % kTcKeyStages;
                        const uint32_t ph = (uint32_t)(i / kTcKeyStages) & 1u;
                        if (!dev::mbar_wait(kempty_bar(s), ph ^ 1u, abort_flag, &g_decode_error, kErrTcProducer)) {
                            ok = false;
                            break;
                        }
                        const uint32_t n = (uint32_t)min((int64_t)kTcTok, sg.t1 - t);
                        dev::mbar_arrive_expect_tx(kfull_bar(s), n * (uint32_t)nw * 4u);
                        dev::bulk_g2s(key_s + (uint32_t)s * kTcKeyBytes, p.kw + r * nw, n * (uint32_t)nw * 4u,
                                      kfull_bar(s));
                    } else {
                        const int s = i % kTcValueStages;
                        const uint32_t ph = (uint32_t)(i / kTcValueStages) & 1u;
                        if (!dev::mbar_wait(vempty_bar(s), ph ^ 1u, abort_flag, &g_decode_error, kErrTcProducer)) {
                            ok = false;
                            break;
                        }
                        dev::mbar_arrive_expect_tx(vfull_bar(s), (uint32_t)kTcVBytes);
                        dev::tma_load_2d(val_s + (uint32_t)s * kTcVBytes, &vmap, vfull_bar(s), 0, (int)r);
                    }
                }
            }
            // never leave the CTA with a copy in flight: wait for the last fill of each stage
            const int stages = keys ? kTcKeyStages : kTcValueStages;
            for (int k = max(0, i - stages); k < i; ++k)
                dev::mbar_drain(keys ? kfull_bar(k % stages) : vfull_bar(k % stages), (uint32_t)(k / stages) & 1u);
            if (keys) dev::mbar_drain(pro_bar, 0);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int c = 0;
            bool ok = true;
            for (int jj = 0; ok && jj < nseg; ++jj) {
                const Segment sg = walk.seg(jj);
                for (int64_t t = sg.t0; t < sg.t1; t += kTcTok, ++c) {
                    const int s = c % kTcValueStages;
                    const uint32_t ph = (uint32_t)(c / kTcValueStages) & 1u;
                    const int a = c % kTcAcc;
                    const uint32_t aph = (uint32_t)(c / kTcAcc) & 1u;
                    if (!dev::mbar_wait(bready_bar(a), aph, abort_flag, &g_decode_error, kErrTcMma) ||
                        !dev::mbar_wait(vfull_bar(s), ph, abort_flag, &g_decode_error, kErrTcMma)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    const uint32_t va = val_s + (uint32_t)s * kTcVBytes;
                    const uint32_t bb = b_s + (uint32_t)a * kTcBBytes;
                    const int nk = (int)((min((int64_t)kTcTok, sg.t1 - t) + 31) / 32);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (k < nk)
                            dev::tc_mma_i8(tmem + (uint32_t)a * 16u, dev::smem_desc_sw128(va + (uint32_t)k * 4096u),
                                           dev::smem_desc_sw128(bb + (uint32_t)k * 32u), kTcIdesc, k > 0 ? 1u : 0u);
                    dev::tc_commit(tfull_bar(a));
                    dev::tc_commit(vempty_bar(s));
                }
            }
            dev::tc_commit(done_bar);
            dev::mbar_drain(done_bar, 0);
        }
    } else if (warp < 2 + kTcScorerWarps) {
        // ---------------- scorers: warp sw takes the chunks c with c % kTcScorerWarps == sw ----------------
        // lane l scores tokens 32 i + l of the chunk, i = 0 .. 3 (MMA slice i), in two pairs
        const int sw = warp - 2;
        const LutLane lut_lane(lane);
        // the byte of token 32 i + lane in row r of B under the 128-byte swizzle:
        // ((2 i + lane / 16) ^ (r % 8)) * 16 + lane % 16, split into a compile-time part
        // and one of two per-lane offsets
        const int bo_even = ((lane >> 4) << 4) + (lane & 15);
        const int bo_odd = (((lane >> 4) ^ 1) << 4) + (lane & 15);
        // The query projections v[g][i] = sum_d S[i][d] q[g][d] (fp32) of every unit this
        // CTA visits, formed once, from S and the queries staged in the table space: thread
        // i (sketch row 32 sw + lane; zero for i >= m) sums its row over the 16-byte column
        // blocks in the rotated order b = (k + lane) % 16, k = 0 .. 15, so that a warp's
        // reads of 32 rows fall in distinct banks.  The first unit's projections build its
        // tables at once; the others wait in this CTA's slots of the workspace (written and
        // read back by the same thread).
        const int row = 32 * sw + lane;
        float* proj = p.sketch_v + (size_t)cta * (size_t)(p.maxj - 1) * G * 256;
        float sv0[G];
        bool ok = __all_sync(0xffffffffu, dev::mbar_wait(pro_bar, 0, abort_flag, &g_decode_error, kErrTcScore));
        if (ok) {
            const uint4* srow = reinterpret_cast<const uint4*>(lut) + row * (kD / 8);
            const uint4* qrows = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(lut) + 65536);
            for (int jj = 0; jj < nseg; ++jj) {
                float sv[G];
#pragma unroll
                for (int g = 0; g < G; ++g) sv[g] = 0.0f;
                if (row < p.m) {
#pragma unroll 4
                    for (int k = 0; k < kD / 8; ++k) {
                        const int blk = (k + lane) & (kD / 8 - 1);
                        const uint4 s8 = srow[blk];
                        const __half2* sh = reinterpret_cast<const __half2*>(&s8);
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const uint4 q8 = qrows[(jj * G + g) * (kD / 8) + blk];
                            const __half2* qh = reinterpret_cast<const __half2*>(&q8);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 a = __half22float2(sh[e]), b = __half22float2(qh[e]);
                                sv[g] = fmaf(a.x, b.x, sv[g]);
                                sv[g] = fmaf(a.y, b.y, sv[g]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    if (jj == 0) sv0[g] = sv[g];
                    else proj[((size_t)(jj - 1) * G + g) * 256 + row] = sv[g];
                }
            }
        }
        // every scorer is done with the staged inputs before the first tables overwrite them
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kTcScorerWarps) : "memory");
        int c = 0;
        for (int jj = 0; jj < nseg; ++jj) {
            const Segment sg = walk.seg(jj);
            const int64_t hb = tc_head0(sg.u);
            // the tables are rebuilt per unit by all scorers; every scorer reaches both
            // barriers, also after an abort (they then skip the work in between)
            if (jj > 0) asm volatile("bar.sync 1, %0;" ::"n"(32 * kTcScorerWarps) : "memory");
            if (ok) {
                float sv[G];
#pragma unroll
                for (int g = 0; g < G; ++g) sv[g] = jj == 0 ? sv0[g] : proj[((size_t)(jj - 1) * G + g) * 256 + row];
                build_sign_tables_from_rows<G>(lut, sv, sw, lane);
            }
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kTcScorerWarps) : "memory");
            for (int64_t t = sg.t0; t < sg.t1; t += kTcTok, ++c) {
                if (!ok || c % kTcScorerWarps != sw) continue;
                const int s = c % kTcKeyStages;
                const uint32_t ph = (uint32_t)(c / kTcKeyStages) & 1u;
                const int a = c % kTcAcc;
                const uint32_t aph = (uint32_t)(c / kTcAcc) & 1u;
                const int n = (int)min((int64_t)kTcTok, sg.t1 - t);
                // the four tokens' norms and value scales straight from global memory
                // (coalesced across the warp; in flight during the table lookups)
                const int64_t r0 = sg.u * p.cap + t;
                uint16_t nrm_b[4];
                float vsc[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool v = 32 * i + lane < n;
                    nrm_b[i] = v ? __ldcs(p.kn + r0 + 32 * i + lane) : (uint16_t)0;
                    vsc[i] = v ? __ldcs(p.vs + r0 + 32 * i + lane) : 0.0f;
                }
                ok = __all_sync(0xffffffffu, dev::mbar_wait(kfull_bar(s), ph, abort_flag, &g_decode_error, kErrTcScore));
                if (!ok) continue;
                const uint8_t* kp = key_p + (size_t)s * kTcKeyBytes;
                float lg[4][G];
#pragma unroll
                for (int pr = 0; pr < 2; ++pr) {
                    uint32_t wA[8], wB[8];
                    const int tA = 64 * pr + lane, tB = tA + 32;
                    if (nw == 8) {
                        const uint4* wp = reinterpret_cast<const uint4*>(kp);
                        const uint4 a0 = wp[2 * tA], a1 = wp[2 * tA + 1], b0 = wp[2 * tB], b1 = wp[2 * tB + 1];
                        wA[0] = a0.x; wA[1] = a0.y; wA[2] = a0.z; wA[3] = a0.w;
                        wA[4] = a1.x; wA[5] = a1.y; wA[6] = a1.z; wA[7] = a1.w;
                        wB[0] = b0.x; wB[1] = b0.y; wB[2] = b0.z; wB[3] = b0.w;
                        wB[4] = b1.x; wB[5] = b1.y; wB[6] = b1.z; wB[7] = b1.w;
                    } else {
                        const uint32_t* wp = reinterpret_cast<const uint32_t*>(kp);
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            wA[k] = k < nw ? wp[tA * nw + k] : 0u;
                            wB[k] = k < nw ? wp[tB * nw + k] : 0u;
                        }
                    }
                    const bool vA = tA < n, vB = tB < n;
                    if (pr == 1) {
                        // the key stage is read: the producer may refill it
                        __syncwarp();
                        if (lane == 0) dev::mbar_arrive(kempty_bar(s));
                    }
                    float scA[G], scB[G];
                    lut_token_sums<G>(wA, lut_s, lut_lane, scA);
                    lut_token_sums<G>(wB, lut_s, lut_lane, scB);
                    const float nA = __half2float(__ushort_as_half(nrm_b[2 * pr]));
                    const float nB = __half2float(__ushort_as_half(nrm_b[2 * pr + 1]));
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float sa = p.qjl_c * nA * scA[g], sb = p.qjl_c * nB * scB[g];
                        lg[2 * pr][g] = vA ? sa * p.scale_log2 : -INFINITY;
                        lg[2 * pr + 1][g] = vB ? sb * p.scale_log2 : -INFINITY;
                        if (p.scores_out != nullptr) {
                            if (vA) p.scores_out[(hb + g) * p.T + t + tA] = sa;
                            if (vB) p.scores_out[(hb + g) * p.T + t + tB] = sb;
                        }
                    }
                }
                // the chunk's max logit per head and max value scale (value scales are >= 0:
                // their bit patterns order like the values); weights 2^(s - Mc) v in fixed
                // point against an exact power of two 2^E with smax 2^E in [2^23, 2^24)
                // (from smax's exponent; chunks whose values are all below 2^-100 count as
                // zero), so the scale itself is not rounded
                float Mc[G];
#pragma unroll
                for (int g = 0; g < G; ++g)
                    Mc[g] = warp_max(fmaxf(fmaxf(lg[0][g], lg[1][g]), fmaxf(lg[2][g], lg[3][g])));
                const uint32_t sexp =
                    __reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fmaxf(vsc[0], vsc[1]), fmaxf(vsc[2], vsc[3])))) >> 23;
                const float rscale = sexp >= 28u ? __uint_as_float((277u - sexp) << 23) : 0.0f;
                uint32_t W[4][G];
                float L[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    uint32_t lq = 0u;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float pe = fast_exp2(lg[i][g] - Mc[g]);   // 0 for an invalid token
                        W[i][g] = min(__float2uint_rn(pe * vsc[i] * rscale), 0xFFFFFFu);
                        lq += __float2uint_rn(pe * 16777216.0f);
                    }
                    L[g] = (float)__reduce_add_sync(0xffffffffu, lq) * 5.9604644775390625e-8f;   // 2^-24
                }
                // operand B and the statistics of buffer a are free once chunk c - kTcAcc is merged
                ok = __all_sync(0xffffffffu, dev::mbar_wait(tempty_bar(a), aph ^ 1u, abort_flag,
                                                            &g_decode_error, kErrTcScore));
                if (!ok) continue;
                uint8_t* bq = b_p + a * kTcBBytes;
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int k = 0; k < 3; ++k) {
                        const int row = 3 * g + k, r7 = row & 7;
                        uint8_t* rp = bq + (row >> 3) * 1024 + r7 * 128 + ((r7 & 1) ? bo_odd : bo_even);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            rp[(((2 * i) ^ r7) & 6) << 4] = (uint8_t)(W[i][g] >> (8 * k));
                    }
                if (lane == 0) {
                    TcChunk& X = chunks[a];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        X.Mc[g] = Mc[g];
                        X.L[g] = L[g];
                    }
                    X.inv = sexp >= 28u ? __uint_as_float((sexp - 23u) << 23) : 0.0f;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) dev::mbar_arrive(bready_bar(a));
            }
        }
    } else if (warp < kTcValueWarp) {
        // ---------------- accumulators: value dimension d ----------------
        const int quarter = warp & 3;
        const int d = quarter * 32 + lane;
        int c = 0;
        bool ok = true;
        for (int jj = 0; ok && jj < nseg; ++jj) {
            const Segment sg = walk.seg(jj);
            float mrun[G], lrun[G], o[G];
#pragma unroll
            for (int g = 0; g < G; ++g) mrun[g] = -INFINITY, lrun[g] = 0.0f, o[g] = 0.0f;
            for (int64_t t = sg.t0; t < sg.t1; t += kTcTok, ++c) {
                const int a = c % kTcAcc;
                const uint32_t aph = (uint32_t)(c / kTcAcc) & 1u;
                // the scorers' arrival on bready publishes the chunk's statistics; the MMA's
                // completion, the accumulators
                ok = __all_sync(0xffffffffu,
                                dev::mbar_wait(bready_bar(a), aph, abort_flag, &g_decode_error, kErrTcAcc) &&
                                    dev::mbar_wait(tfull_bar(a), aph, abort_flag, &g_decode_error, kErrTcAcc));
                if (!ok) break;  // warp-uniform: tcgen05.ld is .aligned
                dev::tc_fence_after();
                // the chunk's statistics and its 16-column accumulator (the four slices summed
                // by the tensor core), then the buffer goes back to the scorers
                const TcChunk& X = chunks[a];
                const float inv = X.inv;
                float Mc[G], num[G], L[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    Mc[g] = X.Mc[g];
                    L[g] = X.L[g];
                }
                {
                    uint32_t r[16];
                    dev::tmem_ld_32x32b_x16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)a * 16u, r);
                    dev::tmem_ld_wait();
                    dev::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) dev::mbar_arrive(tempty_bar(a));
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        // sum_t W c = D2 2^16 + (D1 2^8 + D0): the low part exact in int32
                        // (|.| < 2^31), D2 (|D2| < 2^22) converted exactly through the
                        // 1.5 * 2^23 bias
                        const int lo = (int)r[3 * g + 1] * 256 + (int)r[3 * g];
                        const float d2 = __int_as_float((int)r[3 * g + 2] + 0x4B400000) - kRoundMagic;
                        num[g] = __fmaf_rn(d2, 65536.0f, (float)lo) * inv;
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float mn = fmaxf(mrun[g], Mc[g]);
                    const float al = fast_exp2(mrun[g] - mn);
                    const float be = fast_exp2(Mc[g] - mn);
                    o[g] = __fmaf_rn(o[g], al, num[g] * be);
                    lrun[g] = __fmaf_rn(lrun[g], al, L[g] * be);
                    mrun[g] = mn;
                }
            }
            if (!ok) break;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float* slot = p.ws + (((int64_t)cta * p.maxj + jj) * G + g) * (2 + kD);
                slot[2 + d] = o[g];
                if (d == 0) {
                    slot[0] = mrun[g];
                    slot[1] = lrun[g];
                }
            }
        }
    }

    __syncwarp();  // reconverge warps 0 and 1, whose lane 0 ran the role loop alone
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    if (warp == 1) dev::tmem_dealloc(tmem, kTcTmemCols);
}

// -----------------------------------------------------------------------------------
// INT8 keys and values, both contractions on the tensor cores.  The range streams in
// chunks of 128 tokens of one unit through a key ring and a value ring, each filled by
// TMA tiles (128 rows of 128 bytes, 128-byte swizzle) that its own producer thread issues.
// Per chunk:
//   scores: one tcgen05.mma kind::i8 per 32 dims, D1 [128 tokens x N] = K [128 x 128]
//           (K-major) x Qb^T, where Qb [N x 128 dims] holds, in rows 3 g + k, the base-256
//           digits k (each in -128 .. 127) of the query of head g as a fixed-point integer
//           q_fix = round(q 2^E) with max |q| 2^E in [2^21, 2^22): sum_d c_d q_fix,d =
//           D1[3g] + 2^8 D1[3g+1] + 2^16 D1[3g+2] exactly (|D1| < 2^21 in int32);
//   softmax: four warps, one per 32-token slice (the TMEM lane quarter of its tokens),
//           one token per thread: the logit k_scale 2^-E sum_d c_d q_fix,d * sigma log2 e,
//           the slice's max logit Mc per head, and the weight 2^(s - Mc) v_scale as a
//           24-bit fixed-point integer W against the power of two 2^E' that puts the
//           slice's max value scale into [2^23, 2^24), whose three bytes are rows
//           3 g + k of the value operand B [N x 128 tokens] (K-major); the slice's sum of
//           2^(s - Mc) in 2^-24 fixed point by one integer warp reduction;
//   values: one MMA per slice, D2_i [128 dims x N] = V_i^T [128 x 32 tokens] (MN-major) x
//           W_i^T, each slice into its own accumulator;
//   merge:  four warps, one value dimension per thread: sum_t W_t c_t of each slice (exact
//           in int32), times 2^-E', merged slice by slice into the running online-softmax
//           state of each head.
// Warp roles (one CTA per SM): warp 0 key producer; warp 1 TMEM and the score MMAs; warp
// 2 value producer; warp 3 the value MMAs (each issued as soon as its chunk's weights and
// value tile are in, so that a value stage is held no longer than that); then
// `groups` softmax groups of four warps (group i takes the chunks c with c % groups == i,
// each in its own TMEM and operand buffer i, so that several chunks are scored at once);
// then four merge warps.  The query digits of every unit the CTA visits are formed once,
// at the start, by softmax group 0.
// The products and the per-slice sums are exact; the approximations are the query's
// fixed point (at most 2^-22 max |q| per element), the weights' fixed point (below
// 2^-23 of the slice's max value scale per token), the sums' 2^-24 fixed point, and the
// fp32 rounding of the score and of the merges.
// -----------------------------------------------------------------------------------
constexpr int kI8TcTok = 128;
constexpr int kI8TcKStages = 4;
constexpr int kI8TcVStages = 8;
constexpr int kI8TcMaxUnits = 4;       // units a CTA range may touch (query digits held)
constexpr int kI8TcSoft0 = 4;          // first softmax warp
constexpr int kI8TcTile = kI8TcTok * kD;   // 16 KB

enum : unsigned int { kErrI8TcProducer = 0x221, kErrI8TcMma = 0x222, kErrI8TcSoft = 0x223, kErrI8TcAcc = 0x224 };

template <int G>
struct I8Tc {
    static constexpr int N = G == 8 ? 32 : 16;                // MMA N: rows 3 g + k
    static constexpr int acc = G == 8 ? 2 : 4;                // chunks in flight after their scores
    static constexpr int groups = acc;                        // softmax groups: group i owns buffer i
    static constexpr int acc0 = kI8TcSoft0 + 4 * groups;      // first merge warp
    static constexpr int threads = 32 * (acc0 + 4);
    static constexpr int ob = N * 128;                        // an operand of N rows of 128 bytes
    static constexpr uint32_t cols = 5 * N * acc <= 256 ? 256u : 512u;
    struct Slice {                                            // per chunk and slice
        float Mc[G];                                          // max logit per head (-inf: empty)
        float L[G];                                           // sum of 2^(s - Mc) per head
        float inv;                                            // 2^-E' of the weights
    };
    // shared memory from a 1024-byte aligned base
    static constexpr size_t k_off = 0;
    static constexpr size_t v_off = k_off + (size_t)kI8TcKStages * kI8TcTile;
    static constexpr size_t w_off = v_off + (size_t)kI8TcVStages * kI8TcTile;
    static constexpr size_t q_off = w_off + (size_t)acc * ob;
    static constexpr size_t st_off = q_off + (size_t)kI8TcMaxUnits * ob;
    static constexpr size_t qi_off = st_off + (size_t)acc * 4 * sizeof(Slice);
    static constexpr size_t red_off = qi_off + (size_t)kI8TcMaxUnits * G * sizeof(float);
    static constexpr size_t bar_off = (red_off + 4 * G * sizeof(float) + 7) & ~(size_t)7;
    static constexpr int nbars = 2 * kI8TcKStages + 2 * kI8TcVStages + 5 * acc + 3;
    static constexpr size_t smem = 1024 + bar_off + (size_t)nbars * 8;
    static_assert(smem + 64 <= 232448, "shared memory of one CTA");
    static_assert(w_off % 1024 == 0 && q_off % 1024 == 0 && ob % 1024 == 0, "swizzled operands");
    // instruction descriptors (int32 accumulator, M = 128): scores: A signed K-major,
    // B signed K-major; values: A signed MN-major, B unsigned K-major
    static constexpr uint32_t idesc_qk = (2u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (0u << 16) |
                                         ((uint32_t)(N >> 3) << 17) | ((128u >> 4) << 24);
    static constexpr uint32_t idesc_pv = (2u << 4) | (1u << 7) | (0u << 10) | (1u << 15) | (0u << 16) |
                                         ((uint32_t)(N >> 3) << 17) | ((128u >> 4) << 24);
};

// Byte (row r, column k) of a K-major operand of rows of 128 bytes, 128-byte swizzle.
__device__ __forceinline__ int sw128_byte(int r, int k) {
    const int r7 = r & 7;
    return (r >> 3) * 1024 + r7 * 128 + ((((k >> 4) ^ r7) & 7) << 4) + (k & 15);
}

template <int G>
__global__ void __launch_bounds__(I8Tc<G>::threads, 1)
decode_int8_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap) {
    using C = I8Tc<G>;
    using Slice = typename C::Slice;
    constexpr int N = C::N;
    constexpr int ACC = C::acc;
    extern __shared__ uint8_t i8tc_raw[];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_storage;
    volatile int* abort_flag = &abort_storage;
    const uint32_t raw = dev::smem_u32(i8tc_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* bp = i8tc_raw + (base - raw);
    const uint32_t k_s = base + (uint32_t)C::k_off;
    const uint32_t v_s = base + (uint32_t)C::v_off;
    const uint32_t w_s = base + (uint32_t)C::w_off;
    uint8_t* w_p = bp + C::w_off;
    const uint32_t q_s = base + (uint32_t)C::q_off;
    uint8_t* q_p = bp + C::q_off;
    Slice* slices = reinterpret_cast<Slice*>(bp + C::st_off);       // [ACC][4]
    float* qinv = reinterpret_cast<float*>(bp + C::qi_off);         // [units][G] 2^-E
    float* qred = reinterpret_cast<float*>(bp + C::red_off);        // [4][G]
    const uint32_t bars = base + (uint32_t)C::bar_off;
    auto kfull_bar = [&](int s) { return bars + 8u * s; };
    auto kempty_bar = [&](int s) { return bars + 8u * (kI8TcKStages + s); };
    auto vfull_bar = [&](int s) { return bars + 8u * (2 * kI8TcKStages + s); };
    auto vempty_bar = [&](int s) { return bars + 8u * (2 * kI8TcKStages + kI8TcVStages + s); };
    constexpr int kA0 = 2 * kI8TcKStages + 2 * kI8TcVStages;
    auto sfull_bar = [&](int a) { return bars + 8u * (kA0 + a); };             // scores in TMEM
    auto sempty_bar = [&](int a) { return bars + 8u * (kA0 + ACC + a); };      // scores read
    auto bready_bar = [&](int a) { return bars + 8u * (kA0 + 2 * ACC + a); };  // weights written
    auto tfull_bar = [&](int a) { return bars + 8u * (kA0 + 3 * ACC + a); };   // value sums in TMEM
    auto tempty_bar = [&](int a) { return bars + 8u * (kA0 + 4 * ACC + a); };  // value sums read
    const uint32_t qready_bar = bars + 8u * (kA0 + 5 * ACC);
    const uint32_t done_bar = bars + 8u * (kA0 + 5 * ACC + 1);      // the score MMAs, at the end
    const uint32_t vdone_bar = bars + 8u * (kA0 + 5 * ACC + 2);     // the value MMAs, at the end

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const RangeWalk walk(p, cta / p.nsub);
    const int nseg = walk.count();
    const auto head0 = [&](int64_t u) {
        return (u / p.Hkv) * p.Hq + (u % p.Hkv) * p.Gt + (int64_t)(cta % p.nsub) * G;
    };

    if (threadIdx.x == 0) {
        abort_storage = 0;
        for (int s = 0; s < kI8TcKStages; ++s) {
            dev::mbar_init(kfull_bar(s), 1);
            dev::mbar_init(kempty_bar(s), 1);     // the score MMAs' commit
        }
        for (int s = 0; s < kI8TcVStages; ++s) {
            dev::mbar_init(vfull_bar(s), 1);
            dev::mbar_init(vempty_bar(s), 1);     // the value MMAs' commit
        }
        for (int a = 0; a < ACC; ++a) {
            dev::mbar_init(sfull_bar(a), 1);
            dev::mbar_init(sempty_bar(a), 4);     // the softmax warps
            dev::mbar_init(bready_bar(a), 4);
            dev::mbar_init(tfull_bar(a), 1);
            dev::mbar_init(tempty_bar(a), 4);     // the merge warps
        }
        dev::mbar_init(qready_bar, 1);
        dev::mbar_init(done_bar, 1);
        dev::mbar_init(vdone_bar, 1);
        dev::mbar_init_fence();
    }
    // the operands B (weights and query digits): rows 3 G .. N - 1 stay zero
    for (int i = threadIdx.x; i < (ACC + kI8TcMaxUnits) * C::ob / 16; i += C::threads)
        reinterpret_cast<uint4*>(w_p)[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) dev::tmem_alloc(dev::smem_u32(&tmem_slot), C::cols);
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t tmem_s = tmem;                          // [ACC][N] scores
    const uint32_t tmem_o = tmem + (uint32_t)(ACC * N);    // [ACC][4][N] value sums
    dev::griddep_launch_dependents();  // the combine kernel may be scheduled (it waits)

    if (warp == 0 || warp == 2) {
        // ---------------- producers: warp 0 the key ring, warp 2 the value ring ----------------
        // (KVQ_DECODE_TEST_EXPIRE: the key producer issues nothing, its consumers' waits expire)
        if (lane == 0 && !(warp == 0 && p.test_expire)) {
            const bool keys = warp == 0;
            const CUtensorMap* map = keys ? &kmap : &vmap;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
            const int stages = keys ? kI8TcKStages : kI8TcVStages;
            const uint32_t ring = keys ? k_s : v_s;
            const int err = kErrI8TcProducer;
            int i = 0;
            bool ok = true;
            for (int jj = 0; ok && jj < nseg; ++jj) {
                const Segment sg = walk.seg(jj);
                for (int64_t t = sg.t0; t < sg.t1; t += kI8TcTok, ++i) {
                    const int s = i % stages;
                    const uint32_t ph = (uint32_t)(i / stages) & 1u;
                    const uint32_t full = keys ? kfull_bar(s) : vfull_bar(s);
                    const uint32_t empty = keys ? kempty_bar(s) : vempty_bar(s);
                    if (!dev::mbar_wait(empty, ph ^ 1u, abort_flag, &g_decode_error, err)) {
                        ok = false;
                        break;
                    }
                    dev::mbar_arrive_expect_tx(full, (uint32_t)kI8TcTile);
                    dev::tma_load_2d(ring + (uint32_t)s * kI8TcTile, map, full, 0, (int)(sg.u * p.cap + t));
                }
            }
            // never leave the CTA with a copy in flight: wait for the last fill of each stage
            for (int k = max(0, i - stages); k < i; ++k)
                dev::mbar_drain(keys ? kfull_bar(k % stages) : vfull_bar(k % stages), (uint32_t)(k / stages) & 1u);
        }
    } else if (warp == 1) {
        // ---------------- the score MMAs ----------------
        if (lane == 0) {
            bool ok = dev::mbar_wait(qready_bar, 0u, abort_flag, &g_decode_error, kErrI8TcMma);
            int c = 0;
            for (int jj = 0; ok && jj < nseg; ++jj) {
                const Segment sg = walk.seg(jj);
                for (int64_t t = sg.t0; ok && t < sg.t1; t += kI8TcTok, ++c) {
                    const int a = c % ACC;
                    const int s = c % kI8TcKStages;
                    if (!dev::mbar_wait(sempty_bar(a), ((uint32_t)(c / ACC) & 1u) ^ 1u, abort_flag, &g_decode_error,
                                        kErrI8TcMma) ||
                        !dev::mbar_wait(kfull_bar(s), (uint32_t)(c / kI8TcKStages) & 1u, abort_flag, &g_decode_error,
                                        kErrI8TcMma)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    const uint32_t ka = k_s + (uint32_t)s * kI8TcTile;
                    const uint32_t qb = q_s + (uint32_t)jj * C::ob;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        dev::tc_mma_i8(tmem_s + (uint32_t)(a * N), dev::smem_desc_sw128(ka + (uint32_t)k * 32u),
                                       dev::smem_desc_sw128(qb + (uint32_t)k * 32u), C::idesc_qk, k > 0 ? 1u : 0u);
                    dev::tc_commit(sfull_bar(a));
                    dev::tc_commit(kempty_bar(s));
                }
            }
            dev::tc_commit(done_bar);
            dev::mbar_drain(done_bar, 0);
        }
    } else if (warp == 3) {
        // ---------------- the value MMAs: a chunk's as soon as its weights and values are in ----------------
        if (lane == 0) {
            int j = 0;
            bool ok = true;
            for (int jj = 0; ok && jj < nseg; ++jj) {
                const Segment sg = walk.seg(jj);
                for (int64_t t = sg.t0; ok && t < sg.t1; t += kI8TcTok, ++j) {
                    const int a = j % ACC;
                    const int s = j % kI8TcVStages;
                    if (!dev::mbar_wait(bready_bar(a), (uint32_t)(j / ACC) & 1u, abort_flag, &g_decode_error,
                                        kErrI8TcMma) ||
                        !dev::mbar_wait(vfull_bar(s), (uint32_t)(j / kI8TcVStages) & 1u, abort_flag, &g_decode_error,
                                        kErrI8TcMma)) {
                        ok = false;
                        break;
                    }
                    dev::tc_fence_after();
                    const uint32_t va = v_s + (uint32_t)s * kI8TcTile;
                    const uint32_t wb = w_s + (uint32_t)a * C::ob;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dev::tc_mma_i8(tmem_o + (uint32_t)((a * 4 + i) * N),
                                       dev::smem_desc_sw128(va + (uint32_t)i * 4096u),
                                       dev::smem_desc_sw128(wb + (uint32_t)i * 32u), C::idesc_pv, 0u);
                    dev::tc_commit(tfull_bar(a));
                    dev::tc_commit(vempty_bar(s));
                }
            }
            dev::tc_commit(vdone_bar);
            dev::mbar_drain(vdone_bar, 0);
        }
    } else if (warp < C::acc0) {
        // ---------------- softmax: group grp takes the chunks c with c % groups == grp (its
        // buffer); warp quarter q of the group, token 32 q + lane of the chunk ----------------
        const int q = warp & 3;
        const int grp = (warp - kI8TcSoft0) >> 2;
        const int tid = threadIdx.x - 32 * kI8TcSoft0;     // group 0: 0 .. 127, a query dimension
        // The query digits of every unit, formed once by group 0: thread tid takes dimension
        // tid of the G heads; the max |q| of each head over the 128 dimensions by warp
        // reductions and a pass through shared memory.
        for (int jj = 0; grp == 0 && jj < nseg; ++jj) {
            const int64_t hb = head0(walk.seg(jj).u);
            float qv[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                qv[g] = __half2float(__ushort_as_half(p.q[(hb + g) * kD + tid]));
                const unsigned int m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(qv[g])));
                if (lane == 0) qred[(warp - kI8TcSoft0) * G + g] = __uint_as_float(m);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float amax = fmaxf(fmaxf(qred[g], qred[G + g]), fmaxf(qred[2 * G + g], qred[3 * G + g]));
                // 2^E with amax 2^E in [2^21, 2^22) (fp16 queries: 6 <= E <= 45); all
                // digits zero for a zero query
                const int e = (int)(__float_as_uint(amax) >> 23) - 127;
                const int E = amax > 0.0f ? 21 - e : 0;
                const int qf = __float2int_rn(qv[g] * __uint_as_float((uint32_t)(127 + E) << 23));
                const int d0 = ((qf + 128) & 255) - 128;
                const int r1 = (qf - d0) >> 8;
                const int d1 = ((r1 + 128) & 255) - 128;
                const int d2 = (r1 - d1) >> 8;
                uint8_t* qb = q_p + jj * C::ob;
                qb[sw128_byte(3 * g, tid)] = (uint8_t)d0;
                qb[sw128_byte(3 * g + 1, tid)] = (uint8_t)d1;
                qb[sw128_byte(3 * g + 2, tid)] = (uint8_t)d2;
                if (tid == 0) qinv[jj * G + g] = __uint_as_float((uint32_t)(127 - E) << 23);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        if (grp == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (tid == 0) dev::mbar_arrive(qready_bar);
        }
        // the query scales 2^-E of every unit are in shared memory once the digits are
        bool ok = __all_sync(0xffffffffu, dev::mbar_wait(qready_bar, 0u, abort_flag, &g_decode_error, kErrI8TcSoft));

        const int tl = 32 * q + lane;
        int c = 0;
        for (int jj = 0; jj < nseg; ++jj) {
            const Segment sg = walk.seg(jj);
            const int64_t hb = head0(sg.u);
            float qsc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) qsc[g] = qinv[jj * G + g];
            for (int64_t t = sg.t0; ok && t < sg.t1; t += kI8TcTok, ++c) {
                if (c % C::groups != grp) continue;
                const int a = c % ACC;
                const uint32_t aph = (uint32_t)(c / ACC) & 1u;
                const bool valid = t + tl < sg.t1;
                const int64_t r = sg.u * p.cap + t + tl;
                const float ksc = valid ? __ldcs(p.ks + r) : 0.0f;
                const float vsc = valid ? __ldcs(p.vs + r) : 0.0f;
                ok = __all_sync(0xffffffffu, dev::mbar_wait(sfull_bar(a), aph, abort_flag, &g_decode_error, kErrI8TcSoft));
                if (!ok) break;
                dev::tc_fence_after();
                uint32_t d[N];
                if constexpr (N == 16) dev::tmem_ld_32x32b_x16(tmem_s + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * N), d);
                else dev::tmem_ld_32x32b_x32(tmem_s + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * N), d);
                dev::tmem_ld_wait();
                dev::tc_fence_before();
                __syncwarp();
                if (lane == 0) dev::mbar_arrive(sempty_bar(a));
                float lg[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const int lo = (int)d[3 * g + 1] * 256 + (int)d[3 * g];
                    const float dot = __fmaf_rn((float)(int)d[3 * g + 2], 65536.0f, (float)lo);
                    const float s = dot * (ksc * qsc[g]);
                    lg[g] = valid ? s * p.scale_log2 : -INFINITY;
                    if (p.scores_out != nullptr && valid) p.scores_out[(hb + g) * p.T + t + tl] = s;
                }
                // the slice's max logit per head and max value scale (value scales are
                // >= 0: their bit patterns order like the values); weights in fixed point
                // against 2^E' (from smax's exponent; slices whose values are all below
                // 2^-100 count as zero)
                float Mc[G], L[G];
                uint32_t W[G];
                const uint32_t sexp = __reduce_max_sync(0xffffffffu, __float_as_uint(vsc)) >> 23;
                const float rscale = sexp >= 28u ? __uint_as_float((277u - sexp) << 23) : 0.0f;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    Mc[g] = warp_max(lg[g]);
                    const float pe = valid ? fast_exp2(lg[g] - Mc[g]) : 0.0f;
                    W[g] = min(__float2uint_rn(pe * vsc * rscale), 0xFFFFFFu);
                    L[g] = (float)__reduce_add_sync(0xffffffffu, __float2uint_rn(pe * 16777216.0f)) *
                           5.9604644775390625e-8f;   // 2^-24
                }
                // the weights' buffer and the statistics of buffer a are free once chunk
                // c - ACC is merged
                ok = __all_sync(0xffffffffu,
                                dev::mbar_wait(tempty_bar(a), aph ^ 1u, abort_flag, &g_decode_error, kErrI8TcSoft));
                if (!ok) break;
                uint8_t* wq = w_p + a * C::ob;
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int k = 0; k < 3; ++k) wq[sw128_byte(3 * g + k, tl)] = (uint8_t)(W[g] >> (8 * k));
                if (lane == 0) {
                    Slice& X = slices[a * 4 + q];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        X.Mc[g] = Mc[g];
                        X.L[g] = L[g];
                    }
                    X.inv = sexp >= 28u ? __uint_as_float((sexp - 23u) << 23) : 0.0f;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) dev::mbar_arrive(bready_bar(a));
            }
        }
    } else {
        // ---------------- merge: value dimension d ----------------
        const int quarter = warp & 3;
        const int d = quarter * 32 + lane;
        int c = 0;
        bool ok = true;
        for (int jj = 0; jj < nseg; ++jj) {
            const Segment sg = walk.seg(jj);
            float mrun[G], lrun[G], o[G];
#pragma unroll
            for (int g = 0; g < G; ++g) mrun[g] = -INFINITY, lrun[g] = 0.0f, o[g] = 0.0f;
            for (int64_t t = sg.t0; ok && t < sg.t1; t += kI8TcTok, ++c) {
                const int a = c % ACC;
                const uint32_t aph = (uint32_t)(c / ACC) & 1u;
                // the softmax warps' arrivals on bready publish the statistics; the MMA's
                // completion, the sums
                ok = __all_sync(0xffffffffu,
                                dev::mbar_wait(bready_bar(a), aph, abort_flag, &g_decode_error, kErrI8TcAcc) &&
                                    dev::mbar_wait(tfull_bar(a), aph, abort_flag, &g_decode_error, kErrI8TcAcc));
                if (!ok) break;  // warp-uniform: tcgen05.ld is .aligned
                dev::tc_fence_after();
                const uint32_t ta = tmem_o + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * 4 * N);
                // the four slices' sums, two slices per load
                uint32_t rr[2 * N];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if ((i & 1) == 0) {
                        if constexpr (N == 16) dev::tmem_ld_32x32b_x32(ta + (uint32_t)(i * N), rr);
                        else dev::tmem_ld_32x32b_x64(ta + (uint32_t)(i * N), rr);
                        dev::tmem_ld_wait();
                    }
                    const uint32_t* r = rr + (i & 1) * N;
                    const Slice& X = slices[a * 4 + i];
                    if (X.Mc[0] == -INFINITY) continue;   // a slice without tokens
                    const float inv = X.inv;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const int lo = (int)r[3 * g + 1] * 256 + (int)r[3 * g];
                        const float num = __fmaf_rn((float)(int)r[3 * g + 2], 65536.0f, (float)lo) * inv;
                        const float mc = X.Mc[g];
                        const float mn = fmaxf(mrun[g], mc);
                        const float al = fast_exp2(mrun[g] - mn);
                        const float be = fast_exp2(mc - mn);
                        o[g] = __fmaf_rn(o[g], al, num * be);
                        lrun[g] = __fmaf_rn(lrun[g], al, X.L[g] * be);
                        mrun[g] = mn;
                    }
                }
                // the sums and the statistics are read: buffer a goes back to the softmax warps
                dev::tc_fence_before();
                __syncwarp();
                if (lane == 0) dev::mbar_arrive(tempty_bar(a));
            }
            if (!ok) break;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float* slot = p.ws + (((int64_t)cta * p.maxj + jj) * G + g) * (2 + kD);
                slot[2 + d] = o[g];
                if (d == 0) {
                    slot[0] = mrun[g];
                    slot[1] = lrun[g];
                }
            }
        }
    }

    __syncwarp();  // reconverge warps 0..3, whose lane 0 ran the role loop alone
    dev::tc_fence_before();
    __syncthreads();
    dev::tc_fence_after();
    if (warp == 1) dev::tmem_dealloc(tmem, C::cols);
}

// a / b for non-negative 64-bit a, b > 0, through the 32-bit divide when both fit.
__device__ __forceinline__ int64_t div_nonneg(int64_t a, int64_t b) {
    if (((uint64_t)a | (uint64_t)b) >> 32 == 0) return (int64_t)((uint32_t)a / (uint32_t)b);
    return a / b;
}

// out[b][h][d]: merge, over the token ranges that covered KV unit u = b * Hkv + h / Gt,
// acc_s[d] 2^(m_s - M) / sum_s l_s 2^(m_s - M).  The states of query head h were written by
// the CTAs of its head subgroup (h % Gt) / G, one per range.  If a decode kernel recorded
// an error (a bounded wait gave up and the CTA skipped its work), the states are not
// complete and the head's output is NaN.  Up to eight ranges (the usual case) are read in
// one batch of independent loads, issued together with the error flag's, so the merge
// costs one trip to L2 after the decode kernel drains.
__global__ void __launch_bounds__(kD)
decode_combine_kernel(const float* __restrict__ ws, int64_t T, int64_t W, int maxj, int Hq, int Hkv, int G,
                      int nsub, float* __restrict__ out, float* __restrict__ fin_ml) {
    // Launched as a programmatic dependent of the decode kernel: nothing is read before
    // that kernel has completed and its partial states are visible.
    dev::griddep_wait();
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / Hq;
    const int h = (int)(bh % Hq);
    const int Gt = Hq / Hkv;
    const int64_t u = b * Hkv + h / Gt;
    const int sub = (h % Gt) / G;
    const int gh = h % G;
    const int64_t c0 = div_nonneg(u * T, W);
    const int64_t c1 = div_nonneg((u + 1) * T - 1, W);
    const int d = threadIdx.x;
    auto slot = [&](int64_t c) {
        const int64_t j = u - div_nonneg(c * W, T);
        return ws + (((c * nsub + sub) * maxj + j) * G + gh) * (2 + kD);
    };
    const bool failed = *reinterpret_cast<volatile unsigned int*>(&g_decode_error) != 0u;
    float mx = -INFINITY, l = 0.0f, a = 0.0f;
    if (c1 - c0 < 8) {
        float m8[8], l8[8], a8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k <= c1 - c0) {
                const float* sl = slot(c0 + k);
                m8[k] = sl[0];
                l8[k] = sl[1];
                a8[k] = sl[2 + d];
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k <= c1 - c0) mx = fmaxf(mx, m8[k]);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k <= c1 - c0) {
                const float f = exp2f(m8[k] - mx);
                l += l8[k] * f;
                a += a8[k] * f;
            }
        }
    } else {
        for (int64_t c = c0; c <= c1; ++c) mx = fmaxf(mx, slot(c)[0]);
        for (int64_t c = c0; c <= c1; ++c) {
            const float* sl = slot(c);
            const float f = exp2f(sl[0] - mx);
            l += sl[1] * f;
            a += sl[2 + d] * f;
        }
    }
    if (failed) mx = l = a = __int_as_float(0x7fc00000);
    out[bh * kD + d] = a / l;
    if (fin_ml != nullptr && d == 0) {  // the head's final softmax max (log2 domain) and sum
        fin_ml[2 * bh] = mx;
        fin_ml[2 * bh + 1] = l;
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <int G, bool V4>
size_t int8_smem() {
    return (size_t)I8Ring<G, V4>::stages * I8Ring<G, V4>::bytes +
           (size_t)kI8Consumers * G * (2 + kD) * sizeof(float);
}
constexpr int kQjlThreads = 512;

template <int G, int THREADS = kQjlThreads>
size_t qjl_smem() {
    const size_t tables = (size_t)2 * 256 * 16 * 4 * sizeof(float);   // entries padded to 16 B
    const size_t wbuf = (size_t)(THREADS / 32) * 32 * G * sizeof(float);
    const size_t red = (size_t)(THREADS / 32) * G * (2 + kD) * sizeof(float);
    const size_t a = tables + wbuf;
    return a > red ? a : red;
}

template <int G, bool V4>
cudaError_t run_int8(const DecodeParams& p, int ctas, cudaStream_t st) {
    auto kern = decode_int8_kernel<G, V4>;
    const size_t smem = int8_smem<G, V4>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, kI8Threads, smem, st>>>(p);
    return cudaGetLastError();
}

template <int G, bool RES = false>
size_t qjl_pf_smem() {
    const size_t tables = (size_t)2 * 256 * 16 * 4 * sizeof(float);
    const size_t red = (size_t)kQpfWarps * G * (2 + kD) * sizeof(float);
    const size_t a = (tables > red ? tables : red) + (size_t)kQpfWarps * 32 * G * sizeof(float);
    return a + (size_t)kQpfWarps * kQpfSlot + (RES ? (size_t)G * (kD + 4) * sizeof(float) : 0);
}

template <int G, bool RES = false>
cudaError_t run_qjl_pf(const DecodeParams& p, int ctas, cudaStream_t st) {
    auto kern = decode_qjl_pf_kernel<G, RES>;
    const size_t smem = qjl_pf_smem<G, RES>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, kQpfThreads, smem, st>>>(p);
    return cudaGetLastError();
}

// The tensor-core QJL decode applies when every chunk's copies are 16-byte aligned:
// chunk starts and lengths are multiples of 8 tokens (T and the unit capacity are), the
// arrays are 16-byte aligned, and the value rows fit a TMA row coordinate.
bool qjl_tc_applies(const DecodeParams& p) {
    const auto al16 = [](const void* x) { return reinterpret_cast<uintptr_t>(x) % 16 == 0; };
    const int64_t units = p.T > 0 ? p.total / p.T : 0;
    return !p.cuda_cores && p.knew == nullptr && p.want_out && p.k4p == nullptr && p.m <= 256 && p.m % 32 == 0 &&
           p.maxj <= kTcMaxUnits &&
           p.T % 8 == 0 && p.cap % 8 == 0 && al16(p.kw) && al16(p.vc) && al16(p.q) && al16(p.S) &&
           units * p.cap <= (int64_t)INT32_MAX;
}

// The tensor-core kernel applies and its value map could be made.  That kernel projects
// the queries on the sketch itself; the other QJL kernels read the projections that a
// separate kernel writes to the workspace first.
bool qjl_tc_map(const DecodeParams& p, CUtensorMap* vmap) {
    return qjl_tc_applies(p) && make_u8_rows_map(vmap, p.vc, (p.total / p.T) * p.cap, kTcTok);
}

template <int G>
cudaError_t run_qjl(const DecodeParams& p, int ctas, cudaStream_t st, const CUtensorMap* vmap) {
    if (vmap != nullptr) {
        auto kern = decode_qjl_tc_kernel<G>;
        const size_t smem = tc_smem_bytes();
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<ctas, kTcThreads, smem, st>>>(p, *vmap);
        return cudaGetLastError();
    }
    if (p.knew == nullptr && p.m <= 256) {
        auto kern = decode_qjl_pf_kernel<G>;
        const size_t smem = qjl_pf_smem<G>();
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<ctas, kQpfThreads, smem, st>>>(p);
        return cudaGetLastError();
    }
    auto kern = decode_qjl_kernel<G, kQjlThreads>;
    const size_t smem = qjl_smem<G>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, kQjlThreads, smem, st>>>(p);
    return cudaGetLastError();
}

template <int G>
cudaError_t run_int8_tc_g(const DecodeParams& p, int ctas, cudaStream_t st, const CUtensorMap& kmap,
                          const CUtensorMap& vmap) {
    auto kern = decode_int8_tc_kernel<G>;
    const size_t smem = I8Tc<G>::smem;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, I8Tc<G>::threads, smem, st>>>(p, kmap, vmap);
    return cudaGetLastError();
}

// The tensor-core INT8 kernel for the group size.
cudaError_t run_int8_tc(int G, const DecodeParams& p, int ctas, cudaStream_t st, const CUtensorMap& kmap,
                        const CUtensorMap& vmap) {
    switch (G) {
        case 1: return run_int8_tc_g<1>(p, ctas, st, kmap, vmap);
        case 2: return run_int8_tc_g<2>(p, ctas, st, kmap, vmap);
        case 4: return run_int8_tc_g<4>(p, ctas, st, kmap, vmap);
        case 8: return run_int8_tc_g<8>(p, ctas, st, kmap, vmap);
        default: return cudaErrorNotSupported;
    }
}

// The partial-state kernel for the format and group size; vmap (QJL keys only) selects
// the tensor-core QJL kernel.
cudaError_t run_partial(bool qjl, int G, const DecodeParams& p, int ctas, cudaStream_t st,
                        const CUtensorMap* vmap) {
    if (p.k4p != nullptr) {
        switch (G) {
            case 1: return run_qjl_pf<1, true>(p, ctas, st);
            case 2: return run_qjl_pf<2, true>(p, ctas, st);
            case 4: return run_qjl_pf<4, true>(p, ctas, st);
            default: return cudaErrorNotSupported;
        }
    }
    if (qjl) {
        switch (G) {
            case 1: return run_qjl<1>(p, ctas, st, vmap);
            case 2: return run_qjl<2>(p, ctas, st, vmap);
            case 4: return run_qjl<4>(p, ctas, st, vmap);
            default: return cudaErrorNotSupported;
        }
    }
    if (p.v4p != nullptr) {
        switch (G) {
            case 1: return run_int8<1, true>(p, ctas, st);
            case 2: return run_int8<2, true>(p, ctas, st);
            case 4: return run_int8<4, true>(p, ctas, st);
            case 8: return run_int8<8, true>(p, ctas, st);
            default: return cudaErrorNotSupported;
        }
    }
    switch (G) {
        case 1: return run_int8<1, false>(p, ctas, st);
        case 2: return run_int8<2, false>(p, ctas, st);
        case 4: return run_int8<4, false>(p, ctas, st);
        case 8: return run_int8<8, false>(p, ctas, st);
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

// Query heads one CTA serves per KV head: up to 8 with INT8 keys, up to 4 with QJL keys
// (four 32 KB byte tables fill the shared memory a CTA may use); the largest such
// power of two that divides Hq / Hkv.
int decode_group_size(const kvq_decode_args* a) {
    const int64_t Gt = a->n_q_heads / a->n_kv_heads;
    const int cap = a->key_format == KVQ_KEYS_QJL ? 4 : 8;
    int g = cap;
    while (g > 1 && Gt % g != 0) g >>= 1;
    return g;
}

// The tensor-core INT8 kernel may run this decode: an output, no request for the CUDA
// cores, contexts of at least four chunks, and 16-byte aligned code arrays whose rows a
// TMA coordinate reaches.  (Whether its ranges touch few enough units is checked on the
// plan.)
bool int8_tc_eligible(const kvq_decode_args* a) {
    return a->key_format == KVQ_KEYS_INT8 && a->out != nullptr && (a->flags & KVQ_DECODE_CUDA_CORES) == 0u &&
           a->seq_len >= 4 * kI8TcTok && reinterpret_cast<uintptr_t>(a->k_codes) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(a->v_codes) % 16 == 0 &&
           a->batch * a->n_kv_heads * a->seq_len <= (int64_t)INT32_MAX;
}

DecodePlan plan_decode(const kvq_decode_args* a, int sm_count, bool tc_capable) {
    DecodePlan pl{};
    const int64_t Gt = a->n_q_heads / a->n_kv_heads;
    const int G = decode_group_size(a);
    const bool qjl = a->key_format == KVQ_KEYS_QJL;
    pl.G = G;
    pl.nsub = (int)(Gt / G);
    pl.units = a->batch * a->n_kv_heads;
    const int64_t T = a->seq_len;
    const int64_t total = pl.units * T;
    // The token space is cut into one range per nsub resident CTAs (the CTAs of a range
    // stream the same bytes side by side, each for its own head subgroup).
    const auto cut = [&](int64_t resident) {
        const int64_t ranges = resident / pl.nsub > 0 ? resident / pl.nsub : 1;
        int64_t W = total > 0 ? (total + ranges - 1) / ranges : kRange;
        W = (W + kRange - 1) / kRange * kRange;
        pl.W = W;
        pl.ctas = total > 0 ? (int)((total + W - 1) / W) * pl.nsub : 0;
        pl.maxj = (int)((W + T - 1) / T + 1);
    };
    // As many CTAs as can be resident at once: one tensor-core INT8 CTA per SM (when its
    // ranges touch few enough units), else up to three 68 KB-ring INT8 CTAs per SM, or one
    // QJL CTA per SM (its byte tables fill shared memory).
    // (residual keys run the QJL decode kernel: their key_format is QJL too)
    pl.int8_tc = false;
    if (tc_capable && int8_tc_eligible(a)) {
        cut(sm_count);
        pl.int8_tc = pl.maxj <= kI8TcMaxUnits;
    }
    if (!pl.int8_tc) cut((int64_t)sm_count * (qjl ? 1 : int8_ctas_per_sm(G)));
    pl.partial_bytes = align256((size_t)pl.ctas * pl.maxj * G * (2 + kD) * sizeof(float));
    // QJL: the query projections, or (tensor-core kernel) the slots of the units after a
    // CTA's first
    const size_t proj_pre = (size_t)a->batch * a->n_q_heads * a->sketch_dim;
    const size_t proj_tc = pl.maxj <= kTcMaxUnits ? (size_t)pl.ctas * (size_t)(pl.maxj - 1) * G * 256 : 0;
    const size_t proj = proj_pre > proj_tc ? proj_pre : proj_tc;
    pl.sketch_bytes = qjl ? align256(proj * sizeof(float)) : 0;
    pl.total_bytes = pl.partial_bytes + pl.sketch_bytes;
    return pl;
}

float decode_scale_log2(const kvq_decode_args* a) {
    const float sm = a->sm_scale != 0.0f ? a->sm_scale : 1.0f / sqrtf((float)a->head_dim);
    return sm * kLog2e;
}

cudaError_t launch_decode(const kvq_decode_args* a, const DecodePlan& pl, cudaStream_t st,
                          const AppendSpec* app, const Int4Values* v4, float* fin_ml, const Int4Keys* k4) {
    const int G = pl.G;
    const bool qjl = a->key_format == KVQ_KEYS_QJL;
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
    p.ws = reinterpret_cast<float*>(ws);
    p.sketch_v = qjl ? reinterpret_cast<float*>(ws + pl.partial_bytes) : nullptr;
    p.T = a->seq_len;
    p.cap = app ? app->capacity : a->seq_len;
    p.knew = app ? app->k_new : nullptr;
    p.vnew = (app && a->out) ? app->v_new : nullptr;
    p.S = a->sketch_f16;
    if (v4 != nullptr && a->out != nullptr) {
        p.v4p = v4->packed;
        p.v4s = v4->scales;
        p.v4z = v4->zeros;
        p.v4g = v4->group;
        p.v4_bulk = v4->group == 32 && reinterpret_cast<uintptr_t>(v4->scales) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(v4->zeros) % 16 == 0;
    }
    p.W = pl.W;
    p.total = pl.units * a->seq_len;
    p.Hq = (int)a->n_q_heads;
    p.Hkv = (int)a->n_kv_heads;
    p.Gt = (int)(a->n_q_heads / a->n_kv_heads);
    p.nsub = pl.nsub;
    p.maxj = pl.maxj;
    p.m = qjl ? a->sketch_dim : 0;
    p.scale_log2 = decode_scale_log2(a);
    p.qjl_c = qjl ? (float)(1.2533141373155002512 / (double)a->sketch_dim) : 0.0f;  // sqrt(pi/2)/m
    p.want_out = a->out != nullptr;
    p.cuda_cores = (a->flags & KVQ_DECODE_CUDA_CORES) != 0u;
    p.test_expire = (a->flags & KVQ_DECODE_TEST_EXPIRE) != 0u;
    if (k4 != nullptr) {
        p.k4p = k4->packed;
        p.k4s = k4->scales;
        p.k4z = k4->zeros;
        p.k4_g_shift = k4->group == 32 ? 5 : (k4->group == 64 ? 6 : 7);
        p.k4_ng_shift = 7 - p.k4_g_shift;
    }
    // QJL: value rows are 128 B, so a step's 32 rows start 16-byte aligned whenever the
    // array does
    p.qjl_bulk = qjl && a->out != nullptr && reinterpret_cast<uintptr_t>(a->v_codes) % 16 == 0;
    p.scales_bulk = !qjl && (a->seq_len % 4 == 0) && (p.cap % 4 == 0) &&
                    reinterpret_cast<uintptr_t>(a->k_scales) % 16 == 0 &&
                    (a->out == nullptr || reinterpret_cast<uintptr_t>(a->v_scales) % 16 == 0);
    cudaError_t e;
    if (p.knew != nullptr) {
        // append: where a tensor-core kernel runs the decode, the new token is encoded by
        // a kernel of its own first (the CUDA-core kernels encode it themselves)
        DecodeParams na = p;
        na.knew = nullptr;
        na.vnew = nullptr;
        if (qjl ? qjl_tc_applies(na) : (pl.int8_tc && p.v4p == nullptr)) {
            append_encode_kernel<<<(unsigned)pl.units, qjl ? 32 * (p.m / 32 + 2) : 64, 0, st>>>(p, qjl ? 1 : 0);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            p.knew = nullptr;
            p.vnew = nullptr;
        }
    }
    CUtensorMap vmap;
    const bool tc = qjl && qjl_tc_map(p, &vmap);
    if (qjl && !tc) {
        e = launch_qjl_query_sketch(a->q_f16, a->batch * a->n_q_heads, a->sketch_f16, a->sketch_dim,
                                    const_cast<float*>(p.sketch_v), st);
        if (e != cudaSuccess) return e;
    }
    bool done = false;
    if (pl.int8_tc && p.v4p == nullptr && p.knew == nullptr) {
        CUtensorMap kmap, vmap8;
        const int64_t rows = pl.units * p.cap;
        if (make_u8_rows_map(&kmap, p.kc, rows, kI8TcTok) && make_u8_rows_map(&vmap8, p.vc, rows, kI8TcTok)) {
            e = run_int8_tc(G, p, pl.ctas, st, kmap, vmap8);
            done = true;
        }
    }
    if (!done) e = run_partial(qjl, G, p, pl.ctas, st, tc ? &vmap : nullptr);
    if (e != cudaSuccess || !a->out) return e;
    // The combine kernel is scheduled as the decode kernel's CTAs retire (programmatic
    // dependent launch) instead of after it has fully drained, hiding its launch latency;
    // it waits for the decode kernel before reading the partial states.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a->batch * a->n_q_heads));
    cfg.blockDim = dim3(kD);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float* ws_c = p.ws;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel, ws_c, p.T, p.W, p.maxj, p.Hq, p.Hkv, G, p.nsub,
                              a->out, fin_ml);
}

}  // namespace kvq
