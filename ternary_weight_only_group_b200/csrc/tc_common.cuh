// tc_common.cuh -- device helpers shared by the tensor-core kernels (sm_100a):
// mbarriers with bounded waits, TMA loads, UMMA descriptors, tcgen05 MMA /
// commit / fences / TMEM loads, and the on-chip ternary decoder that writes
// bf16 weights into the 128-byte-swizzled K-major layout.
#pragma once

#include <cuda.h>

#include <cstdlib>

#include "tq_internal.cuh"

namespace tq {
namespace tc {

constexpr uint64_t kTimeoutNs = 2000000000ull;  // default bound of every mbarrier wait: 2 s

// Bound of the kernels' mbarrier waits, and a test hook: with withhold_x set,
// the TMA producer of every CTA leaves out its first activation load, so the
// consumer waiting for it gives up after limit_ns (TQ_DERR_TIMEOUT) and the
// whole CTA winds down through the abort path.  Read from the environment at
// every launch (TQ_DEBUG_WAIT_LIMIT_NS, TQ_DEBUG_WITHHOLD_X_LOAD); unset, the
// limit is 2 s and nothing is withheld.
struct WaitCfg {
    uint64_t limit_ns;
    int withhold_x;
};

inline WaitCfg wait_cfg_from_env() {
    WaitCfg w{kTimeoutNs, 0};
    if (const char* e = getenv("TQ_DEBUG_WAIT_LIMIT_NS")) {
        const unsigned long long v = strtoull(e, nullptr, 10);
        if (v > 0 && v < kTimeoutNs) w.limit_ns = v;
    }
    if (const char* e = getenv("TQ_DEBUG_WITHHOLD_X_LOAD")) w.withhold_x = atoi(e) != 0;
    return w;
}

__device__ __forceinline__ uint32_t s32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(s32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false when the deadline (limit ns) passed or another role gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, uint64_t limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            s32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(s32(bar))
        : "memory");
}

// Shared-memory matrix descriptor, K-major operand with 128-byte swizzle:
// rows of 128 bytes, 8-row atoms 1024 bytes apart (SBO), version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;             // leading byte offset (16 B; unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: 1024 B between 8-row groups
    d |= (uint64_t)1 << 46;             // descriptor version
    d |= (uint64_t)2 << 61;             // SWIZZLE_128B
    return d;
}

// Instruction descriptor: kind::f16, bf16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// The same MMA with A read from tensor memory (rows in lanes 0..127, two bf16
// of a row per 32-bit column, K order), B from shared memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(s32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 consecutive columns of this thread's lane (warp quadrant's 32 lanes),
// followed by the wait for the stores to land.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 16 consecutive columns of this thread's lane, then the wait for the stores.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Code bytes q_lo .. q_lo+13 of one row for a stage, read from the staged
// 32-byte window (TMA mode): the window starts at the 16-byte-aligned byte at
// or below the first needed one, `off` bytes earlier.
__device__ __forceinline__ void window_bytes(const uint8_t* row32, int off, uint32_t (&bytes)[14]) {
    const uint4 lo = *reinterpret_cast<const uint4*>(row32);
    const uint4 hi = *reinterpret_cast<const uint4*>(row32 + 16);
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    const uint32_t sh = (uint32_t)(off & 3) * 8u;
    uint32_t o[4];
    switch (off >> 2) {
        case 0:
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = __funnelshift_r(w[i], w[i + 1], sh);
            break;
        case 1:
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = __funnelshift_r(w[i + 1], w[i + 2], sh);
            break;
        case 2:
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = __funnelshift_r(w[i + 2], w[i + 3], sh);
            break;
        default:
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = __funnelshift_r(w[i + 3], w[i + 4], sh);
            break;
    }
#pragma unroll
    for (int i = 0; i < 14; ++i) bytes[i] = (o[i >> 2] >> (8 * (i & 3))) & 0xFFu;
}


// Single-path decoder of one row's 64 weights for a stage: columns c0 ..
// c0+63 of one group, c0 a multiple of 64, r0 = c0 % 5.  bytes[] holds code
// bytes q_lo = c0 / 5 .. q_lo + 13 of the group (those past the group only
// feed digits past the stage, so their values do not matter).  When the
// stage holds the group's last byte (check_pad), `lastb` is that byte, and a
// canonical one lies in [pad_base, pad_base + pad_span).  `lut4` maps a byte
// to the PRMT selectors of its digits 0..3 (digit d -> 0x10 + 0x22 d over
// V = {-s, 0}, Z = {+s, NaN}; bytes >= 243 select NaN); digit 4 is
// floor(b / 81) = (b * 810) >> 16, exact for every byte, and 3 (NaN) for
// b >= 243.  Four-byte entries halve the bank conflicts of the lookups.  The selector stream of the 14
// bytes is packed into words by PRMT and funnel-shifted by r0 bytes, so every
// stage takes the same code.  A rejected scale or padding digit makes the
// row's stage NaN.  Writes the 128-byte swizzled K-major tile row.
// `put(k, v)` receives the decoded columns 8k .. 8k+7 as four bf16 pairs.
template <int LUT_STRIDE, class Put>
__device__ __forceinline__ void decode_stage64_to(const uint32_t* lut4, const uint32_t (&bytes)[14], int r0,
                                                  bool check_pad, uint32_t lastb, uint32_t pad_base,
                                                  uint32_t pad_span, uint32_t scale_bits, Put&& put) {
    uint2 e[14];
#pragma unroll
    for (int i = 0; i < 14; ++i) {
        const uint32_t b = bytes[i] & 0xFFu;
        e[i].x = lut4[b * LUT_STRIDE];               // selectors of digits 0..3
        e[i].y = 0x10u + 0x22u * ((b * 810u) >> 16);  // digit 4 = floor(b / 81), 3 for b >= 243
    }
    uint32_t W[17];
#pragma unroll
    for (int h = 0; h < 3; ++h) {
        const uint2 a = e[4 * h], b = e[4 * h + 1], c = e[4 * h + 2], d = e[4 * h + 3];
        W[5 * h + 0] = a.x;
        W[5 * h + 1] = prmt(a.y, b.x, 0x6540u);
        W[5 * h + 2] = prmt(prmt(b.x, b.y, 0x0043u), c.x, 0x5410u);
        W[5 * h + 3] = prmt(prmt(c.x, c.y, 0x0432u), d.x, 0x4210u);
        W[5 * h + 4] = prmt(d.x, d.y, 0x4321u);
    }
    W[15] = e[12].x;
    W[16] = prmt(e[12].y, e[13].x, 0x6540u);
    bool bad = scale_is_bad(scale_bits);
    if (check_pad) bad |= lastb - pad_base >= pad_span;
    uint32_t V, Z;
    if (bad) {
        V = Z = 0x7FC07FC0u;
    } else {
        const uint32_t mag = scale_bits == 0 ? 0u : scale_to_bf16_bits((uint16_t)scale_bits);
        V = mag ? (mag | 0x8000u) : 0u;  // {-s, 0}
        Z = mag | 0x7FC00000u;           // {+s, NaN}
    }
    const uint32_t sh = 8u * (uint32_t)r0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t o0 = __funnelshift_rc(W[2 * k], W[2 * k + 1], sh);
        const uint32_t o1 = __funnelshift_rc(W[2 * k + 1], W[2 * k + 2], sh);
        put(k, make_uint4(prmt(V, Z, o0), prmt(V, Z, o0 >> 16), prmt(V, Z, o1), prmt(V, Z, o1 >> 16)));
    }
}
template <int LUT_STRIDE = 1>
__device__ __forceinline__ void decode_stage64(const uint32_t* lut4, const uint32_t (&bytes)[14], int r0,
                                               bool check_pad, uint32_t lastb, uint32_t pad_base,
                                               uint32_t pad_span, uint32_t scale_bits, uint8_t* tile_row,
                                               int row_in_atom) {
    decode_stage64_to<LUT_STRIDE>(lut4, bytes, r0, check_pad, lastb, pad_base, pad_span, scale_bits,
                                  [&](int k, uint4 v) { *reinterpret_cast<uint4*>(tile_row + ((k ^ row_in_atom) << 4)) = v; });
}

// Decoder of one row's 64 weights for a stage in the 2-bit format (code c =
// t + 1 of weight j in bits 2 (j mod 4) of byte j / 4; code 3 invalid): the
// four 32-bit words w[] hold the stage's 64 codes in column order (G a
// multiple of 64, so the stage lies in one group and has no padding).
// (w >> 2k) & 0x03030303 holds the codes of columns k, k+4, k+8, k+12 in its
// bytes; mapped to selector bytes 0x10 + 0x22 c over V = {-s, 0}, Z = {+s,
// NaN} and interleaved by PRMT into the selector pairs of adjacent columns,
// one PRMT per column pair picks the bf16 values.  Code 3 and a rejected
// scale give NaN.  Writes the 128-byte swizzled K-major tile row.
template <class Put>
__device__ __forceinline__ void decode_stage64_2bit_to(const uint32_t (&w)[4], uint32_t scale_bits, Put&& put) {
    uint32_t V, Z;
    if (scale_is_bad(scale_bits)) {
        V = Z = 0x7FC07FC0u;
    } else {
        const uint32_t mag = scale_bits == 0 ? 0u : scale_to_bf16_bits((uint16_t)scale_bits);
        V = mag ? (mag | 0x8000u) : 0u;  // {-s, 0}
        Z = mag | 0x7FC00000u;           // {+s, NaN}
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // columns 16 q .. 16 q + 15
        uint32_t s[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) s[k] = 0x10101010u + 0x22u * ((w[q] >> (2 * k)) & 0x03030303u);
        const uint32_t p01a = prmt(s[0], s[1], 0x5140u);  // columns (0,1) low half, (4,5) high half
        const uint32_t p23a = prmt(s[2], s[3], 0x5140u);  // (2,3), (6,7)
        const uint32_t p01b = prmt(s[0], s[1], 0x7362u);  // (8,9), (12,13)
        const uint32_t p23b = prmt(s[2], s[3], 0x7362u);  // (10,11), (14,15)
        put(2 * q, make_uint4(prmt(V, Z, p01a), prmt(V, Z, p23a), prmt(V, Z, p01a >> 16), prmt(V, Z, p23a >> 16)));
        put(2 * q + 1,
            make_uint4(prmt(V, Z, p01b), prmt(V, Z, p23b), prmt(V, Z, p01b >> 16), prmt(V, Z, p23b >> 16)));
    }
}
__device__ __forceinline__ void decode_stage64_2bit(const uint32_t (&w)[4], uint32_t scale_bits, uint8_t* tile_row,
                                                    int row_in_atom) {
    decode_stage64_2bit_to(w, scale_bits,
                           [&](int k, uint4 v) { *reinterpret_cast<uint4*>(tile_row + ((k ^ row_in_atom) << 4)) = v; });
}

// Canonical range of a group's last code byte: digits REAL..4 equal to 1,
// i.e. [base, base + 3^REAL) with base = sum_{i=REAL}^{4} 3^i (REAL < 5);
// every byte below 243 when REAL == 5.
__host__ __device__ inline void padding_range(int G, uint32_t& base, uint32_t& span) {
    const int B = bytes_per_group(G);
    const int real = G - 5 * (B - 1);
    uint32_t b = 0, p = 1;
    for (int i = 0; i < 5; ++i) {
        if (i >= real) b += p;
        p *= 3;
    }
    uint32_t sp = 1;
    for (int i = 0; i < real; ++i) sp *= 3;
    base = b;
    span = sp;
}

// Encoder of 2-D TMA descriptors (driver entry point, no libcuda link).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, void* base, uint64_t dim0, uint64_t dim1,
                    uint64_t stride1_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle swizzle);

}  // namespace tc
}  // namespace tq
