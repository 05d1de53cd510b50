// tq_internal.cuh -- device helpers shared by the libtq kernels (CUDA side only).
//
// Format facts used here come from "precisit/pack-unpack-run" (codec.py
// description): one binary16 scale per group of G columns, five base-3 digits
// per byte, each group byte-aligned, digit d = t + 1, first weight = least
// significant digit, padding digit 1, bytes >= 243 invalid.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "tq.h"

namespace tq {

// Split cluster barrier.  Every thread of every CTA of the cluster arrives
// once (relaxed) and later waits; once the wait returns, all CTAs of the
// cluster are known to be running, so their shared memory may be written
// through distributed shared memory.  Both calls must be reached by all
// threads, warp-converged.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Packed fp32 pairs (sm_100: one instruction adds or fuses both lanes of a pair).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// A kernel's dynamic shared-memory limit, raised on demand and never lowered:
// the check and the raise happen under one lock, so two host threads asking
// for different sizes cannot leave the attribute below what either launches.
struct SmemAttr {
    std::mutex mu;
    std::atomic<int> cur{0};
    template <typename Kern>
    cudaError_t ensure(Kern kern, int bytes) {
        if (bytes <= cur.load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lk(mu);
        if (bytes <= cur.load(std::memory_order_relaxed)) return cudaSuccess;
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e == cudaSuccess) cur.store(bytes, std::memory_order_release);
        return e;
    }
};

__host__ __device__ constexpr int bytes_per_group(int G) { return (G + 4) / 5; }

// Byte of a group made only of zero trits: 1 + 3 + 9 + 27 + 81.
constexpr uint32_t kZeroByte = 121;
// bf16 bit pattern written for a rejected group.
constexpr uint16_t kBf16NaN = 0x7FC0;
// Largest bf16 magnitude pattern whose group mean is certain to round to +0:
// max|w| <= 2^-25 implies mean <= 2^-25, the tie below the smallest binary16
// subnormal, which rounds to even (+0).
constexpr uint32_t kTinyMaxBits = 0x3300;  // bf16 2^-25
// bf16 pattern of 2^32: a magnitude at or above it makes any group mean
// (G <= 4096) exceed 65520 and overflow binary16.
constexpr uint32_t kHugeBits = 0x4F80;

__device__ __forceinline__ uint32_t seg_max_u32(uint32_t v, int width) {
    for (int off = width >> 1; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}
__device__ __forceinline__ uint32_t seg_or_u32(uint32_t v, int width) {
    for (int off = width >> 1; off > 0; off >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}
__device__ __forceinline__ double seg_sum_f64(double v, int width) {
    for (int off = width >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Exact binary64 value of a normal bf16 magnitude pattern a (1 <= exponent <= 254):
// same exponent, the 7 fraction bits moved to the top of the 52-bit fraction.
__device__ __forceinline__ double bf16_normal_mag_to_f64(uint32_t a) {
    return __hiloint2double((int)((a << 13) + 0x38000000u), 0);
}

// RNE bf16 of a binary16 scale, as the decoded magnitude of a nonzero trit.
__device__ __forceinline__ uint16_t scale_to_bf16_bits(uint16_t s) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(__half2float(__ushort_as_half(s))));
}

// True for a stored scale the decoder must reject: sign bit set, or NaN/Inf.
__device__ __forceinline__ bool scale_is_bad(uint32_t s) {
    return (s & 0x8000u) != 0 || (s & 0x7C00u) == 0x7C00u;
}

// Trit threshold: |w| > s/2  <=>  (|w| bf16 pattern) > (binary32 pattern of s/2) >> 16.
// Both sides are non-negative floats, whose order is the order of their bit
// patterns; a bf16 pattern shifted left by 16 is the binary32 of the same value.
// A zero scale gives a threshold no magnitude exceeds.
__device__ __forceinline__ uint32_t trit_threshold(uint16_t s) {
    if (s == 0) return 0xFFFFu;
    float half_s = __half2float(__ushort_as_half(s)) * 0.5f;  // exact
    return __float_as_uint(half_s) >> 16;
}

// ---------------------------------------------------------------------------
// Exact group scale by multi-word integer arithmetic (any G <= TQ_MAX_G, any
// exponent spread).  The sum of |w| is held exactly in units of 2^-133 (the
// smallest bf16 subnormal); it is divided by G and rounded once to binary16,
// ties to even.  Returns TQ_DERR_* bits; *s_out is +0 on error.
// ---------------------------------------------------------------------------
static __device__ __noinline__ uint32_t exact_group_scale(const uint16_t* __restrict__ w, int G,
                                                    uint16_t* s_out) {
    *s_out = 0;
    uint32_t amax = 0;
    // Every magnitude below 2^32 (kHugeBits) is below 2^165 units; G <= 2^12
    // of them fit in 6 words.  Larger ones (and Inf/NaN) only decide the error
    // below, so they are not added.
    uint32_t L[6] = {0, 0, 0, 0, 0, 0};
    auto add = [&](uint32_t a) {
        amax = max(amax, a);
        if (a >= kHugeBits) return;
        uint32_t e = a >> 7;
        uint32_t m = (a & 0x7F) | (e ? 0x80u : 0u);
        uint32_t sh = e ? e - 1 : 0;
        uint32_t limb = sh >> 5, bit = sh & 31;
        uint64_t v = (uint64_t)m << bit;
        uint64_t carry = 0;
        for (uint32_t i = limb; i < 6; ++i) {
            uint64_t t = (uint64_t)L[i] + (v & 0xFFFFFFFFull) + carry;
            L[i] = (uint32_t)t;
            carry = t >> 32;
            v >>= 32;
            if (v == 0 && carry == 0) break;
        }
    };
    if ((reinterpret_cast<uintptr_t>(w) & 15) == 0 && G % 8 == 0) {
        // 16-byte loads, four in flight: the group costs a few load latencies, not G
        for (int j = 0; j < G; j += 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = j + 8 * u < G ? __ldg(reinterpret_cast<const uint4*>(w + j + 8 * u)) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t h[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int k = 0; k < 8; ++k) add((h[k >> 1] >> (16 * (k & 1))) & 0x7FFFu);
            }
        }
    } else {
        for (int j = 0; j < G; ++j) add(w[j] & 0x7FFFu);
    }
    if (amax >= 0x7F80u) return TQ_DERR_WEIGHT;
    if (amax >= kHugeBits) return TQ_DERR_OVERFLOW;
    if (amax <= kTinyMaxBits) return 0;
    uint32_t Q[6];
    uint64_t r = 0;
    for (int i = 5; i >= 0; --i) {
        uint64_t cur = (r << 32) | L[i];
        Q[i] = (uint32_t)(cur / (uint32_t)G);
        r = cur % (uint32_t)G;
    }
    int P = -1;
    for (int i = 5; i >= 0; --i)
        if (Q[i]) { P = i * 32 + 31 - __clz(Q[i]); break; }
    if (P < 0) return 0;
    int E = P - 133;  // floor(log2(mean))
    if (E > 15) return TQ_DERR_OVERFLOW;
    int Eeff = E < -14 ? -14 : E;
    int k = Eeff + 123;  // one binary16 ulp is 2^k units
    auto bit_of = [&](int b) -> uint32_t { return (Q[b >> 5] >> (b & 31)) & 1u; };
    uint32_t mant = 0;
    for (int i = 0; i < 12; ++i) mant |= bit_of(k + i) << i;
    uint32_t half = bit_of(k - 1);
    bool rest = (r != 0);
    for (int b = 0; b < k - 1 && !rest; ++b) rest = bit_of(b) != 0;
    uint32_t up = half && (rest || (mant & 1u));
    uint32_t bits = ((uint32_t)(Eeff + 14) << 10) + mant + up;
    if (bits >= 0x7C00u) return TQ_DERR_OVERFLOW;
    *s_out = (uint16_t)bits;
    return 0;
}

// Decode table entry for a byte: its five digits, 2 bits each (digit i at
// bits 2i..2i+1), with bit 15 set for an invalid byte (>= 243).
__device__ __forceinline__ uint32_t byte_digit_pattern(uint32_t b) {
    if (b >= 243) return 0x8000u;
    uint32_t p = 0;
    for (int i = 0; i < 5; ++i) {
        p |= (b % 3) << (2 * i);
        b /= 3;
    }
    return p;
}

// Digit pattern of a canonical last byte: digits >= `real` are all 1.
__host__ __device__ constexpr uint32_t padding_mask(int real) { return 0x3FFu & ~((1u << (2 * real)) - 1u); }
__host__ __device__ constexpr uint32_t padding_ones(int real) { return 0x155u & padding_mask(real); }

// PRMT selector byte of a digit d: the bf16 value of a weight is picked from
// the 8 bytes {V, Z} = {-s, 0, +s, NaN}; digit d (d = t + 1) selects bytes
// 2d and 2d+1, i.e. selector 0x10 + 0x22 d, and d = 3 (invalid) selects NaN.
__device__ __forceinline__ uint32_t digit_selector(uint32_t d) { return 0x10u + 0x22u * d; }

__device__ __forceinline__ uint32_t prmt32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// Selector bytes of the 8 consecutive weights p0 .. p0+7 of a group (p0 % 8
// == 0) from the code bytes b0, b1, b2 holding them (weight p0 is digit
// r = p0 % 5 of b0) and a byte -> selectors table; invalid bytes select NaN.
__device__ __forceinline__ void eight_selectors(const uint2* sel_lut, uint32_t b0, uint32_t b1, uint32_t b2,
                                                uint32_t shift, uint32_t& o0, uint32_t& o1) {
    const uint2 e0 = sel_lut[b0], e1 = sel_lut[b1], e2 = sel_lut[b2];
    const uint32_t w0 = e0.x;                                                // s0..s3
    const uint32_t w1 = prmt32(e0.y, e1.x, 0x6540u);                         // s4..s7
    const uint32_t w2 = prmt32(prmt32(e1.x, e1.y, 0x4343u), e2.x, 0x5410u);  // s8..s11
    o0 = __funnelshift_rc(w0, w1, shift);
    o1 = __funnelshift_rc(w1, w2, shift);
}

// Fills a byte -> selector-bytes table (digit i in byte i) for the {-s, 0, +s, NaN} layout.
// Selectors of digits 0..3 of every byte (bytes >= 243: all NaN).
__device__ __forceinline__ uint32_t digit_selector_word4(uint32_t b) {
    uint32_t w = 0, v = b;
    for (int i = 0; i < 4; ++i) {
        w |= digit_selector(b >= 243 ? 3u : v % 3u) << (8 * i);
        v /= 3u;
    }
    return w;
}

__device__ __forceinline__ void fill_digit_selector_lut4(uint32_t* lut4, int tid, int nthreads) {
    for (int b = tid; b < 256; b += nthreads) lut4[b] = digit_selector_word4((uint32_t)b);
}

// The same table held once per lane: word b * 32 + lane (bank `lane`), so
// the 32 lookups of a warp never conflict, whatever the bytes.  32 KB.  Every
// thread of the block calls it (whole warps; blockDim a multiple of 32): warp
// w computes the words of bytes 32w .. 32w+31, one per lane, and stores each
// byte's 32 copies with one conflict-free store.
__device__ __forceinline__ void fill_digit_selector_lut4_lanes(uint32_t* lut, int tid, int nthreads) {
    const int ln = tid & 31;
    for (int b0 = (tid >> 5) * 32; b0 < 256; b0 += (nthreads >> 5) * 32) {
        const uint32_t mine = digit_selector_word4((uint32_t)(b0 + ln));
#pragma unroll 8
        for (int j = 0; j < 32; ++j) lut[(b0 + j) * 32 + ln] = __shfl_sync(0xFFFFFFFFu, mine, j);
    }
}

__device__ __forceinline__ void fill_digit_selector_lut(uint2* sel_lut, int tid, int nthreads) {
    for (int b = tid; b < 256; b += nthreads) {
        uint32_t sv[5];
        uint32_t v = b;
        for (int i = 0; i < 5; ++i) {
            sv[i] = digit_selector(b >= 243 ? 3u : v % 3);
            v /= 3;
        }
        sel_lut[b] = make_uint2(sv[0] | (sv[1] << 8) | (sv[2] << 16) | (sv[3] << 24), sv[4]);
    }
}

// Error bits of one weight row (its ng groups of B code bytes and ng scales);
// the GEMV kernels call it only for an output row that came out NaN.
static __device__ __noinline__ uint32_t scan_row_errors(const uint8_t* crow, const uint16_t* srow, int ng, int G, int B) {
    const int real = G - 5 * (B - 1);
    const uint32_t pm = padding_mask(real), po = padding_ones(real);
    uint32_t bad = 0;
    for (int g = 0; g < ng; ++g) {
        if (scale_is_bad(srow[g])) bad |= TQ_DERR_SCALE;
        for (int q = 0; q < B; ++q) {
            const uint32_t p = byte_digit_pattern(crow[g * B + q]);
            if (p & 0x8000u) bad |= TQ_DERR_BYTE;
            else if (q == B - 1 && (p & pm) != po) bad |= TQ_DERR_PADDING;
        }
    }
    return bad;
}

// The same for the 2-bit format (ceil(G/4) bytes per group, code c in bits
// 2 (j mod 4) of byte j / 4): a code 3 sets TQ_DERR_BYTE (a padding position
// included), a padding code other than 1 or 3 TQ_DERR_PADDING.
static __device__ __noinline__ uint32_t scan_row_errors2(const uint8_t* crow, const uint16_t* srow, int ng, int G) {
    const int B = (G + 3) / 4;
    uint32_t bad = 0;
    for (int g = 0; g < ng; ++g) {
        if (scale_is_bad(srow[g])) bad |= TQ_DERR_SCALE;
        for (int j = 0; j < 4 * B; ++j) {
            const uint32_t c = (crow[g * B + j / 4] >> (2 * (j % 4))) & 3u;
            if (c == 3u) bad |= TQ_DERR_BYTE;
            else if (j >= G && c != 1u) bad |= TQ_DERR_PADDING;
        }
    }
    return bad;
}

}  // namespace tq
