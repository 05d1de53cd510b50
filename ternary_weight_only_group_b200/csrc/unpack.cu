// unpack.cu -- base-3 decoder to bf16.
//
// "precisit/pack-unpack-run", codec.py description: the decoder turns codes
// back into bf16 weights and treats byte values from 243 up as invalid; the
// paragraph after it: a scale stored as zero decodes its whole group to 0.
//
// Fast path (G = 8 * 2^k, 8 <= G <= 256): G/8 lanes per group, each lane
// writes 8 consecutive bf16 with one 16-byte store.  Each lane checks the
// code bytes it loads (>= 243 invalid; the group's last byte against the
// canonical padding range), the verdicts are OR-ed across the group's lanes,
// and a rejected group is written as bf16 NaN.  Selectors come from a
// 256-entry shared-memory table.
#include "tq_internal.cuh"

namespace tq {

template <int G>
__global__ void __launch_bounds__(256) unpack_pow2_kernel(
    const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales, int64_t num_groups,
    uint16_t* __restrict__ out, uint32_t* __restrict__ d_err) {
    constexpr int LPG = G / 8;
    constexpr int GPW = 32 / LPG;
    constexpr int B = bytes_per_group(G);
    constexpr int REAL = G - 5 * (B - 1);  // real digits in the last byte (1..5)
    // a canonical last byte has digits REAL..4 equal to 1: [PAD_BASE, PAD_BASE + 3^REAL)
    constexpr uint32_t PAD_SPAN = REAL == 1 ? 3u : (REAL == 2 ? 9u : (REAL == 3 ? 27u : 81u));
    constexpr uint32_t PAD_BASE = REAL == 1 ? 120u : (REAL == 2 ? 117u : (REAL == 3 ? 108u : 81u));
    __shared__ uint2 sel_lut[256];
    fill_digit_selector_lut(sel_lut, threadIdx.x, blockDim.x);
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int sub = lane % LPG;
    const int p0 = 8 * sub;
    const int q_first = p0 / 5;      // byte holding weight p0
    const int r_first = p0 - 5 * q_first;
    const uint32_t shift = 8u * (uint32_t)r_first;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    uint32_t err_acc = 0;

    // weights p0..p0+7 lie in bytes q_first .. q_first+2 (the third only for its
    // first digits); the next pass's bytes and scale are loaded before this
    // pass is decoded
    const int64_t stride = nwarps * GPW;
    auto load = [&](int64_t base, uint32_t (&bv)[3], uint32_t& s) {
        const int64_t gi = base + lane / LPG;
        bv[0] = bv[1] = bv[2] = kZeroByte;
        s = 0;
        if (gi < num_groups) {
            const uint8_t* in = codes + gi * B;
#pragma unroll
            for (int t = 0; t < 3; ++t)
                if (q_first + t < B) bv[t] = __ldcs(in + q_first + t);
            s = __ldg(scales + gi);
        }
    };
    uint32_t bv_next[3], s_next;
    load(warp * GPW, bv_next, s_next);
    for (int64_t base = warp * GPW; base < num_groups; base += stride) {
        const int64_t gi = base + lane / LPG;
        const bool active = gi < num_groups;
        const uint32_t bv[3] = {bv_next[0], bv_next[1], bv_next[2]};
        const uint32_t s = s_next;
        load(base + stride, bv_next, s_next);
        // validation of the lane's bytes (a byte seen by two lanes is checked
        // twice; the verdicts are OR-ed): >= 243 is invalid; the group's last
        // byte must lie in [PAD_BASE, PAD_BASE + PAD_SPAN) (padding digits 1)
        uint32_t bad = 0;
#pragma unroll
        for (int t = 0; t < 3; ++t) {
            const uint32_t b = bv[t];  // 121 (valid) past the group
            if (b >= 243) bad |= TQ_DERR_BYTE;
            else if (REAL < 5 && q_first + t == B - 1 && b - PAD_BASE >= PAD_SPAN) bad |= TQ_DERR_PADDING;
        }
        if (sub == 0 && scale_is_bad(s)) bad |= TQ_DERR_SCALE;
        bad = seg_or_u32(bad, LPG);
        if (!active) bad = 0;

        uint32_t o0, o1;  // selector bytes of the lane's 8 weights
        eight_selectors(sel_lut, bv[0], bv[1], bv[2], shift, o0, o1);
        uint32_t V, Z;  // {-s, 0} and {+s, NaN}
        if (bad) {
            V = Z = 0x7FC07FC0u;
        } else {
            const uint32_t mag = (s == 0) ? 0u : scale_to_bf16_bits((uint16_t)s);
            V = mag ? (mag | 0x8000u) : 0u;
            Z = mag | 0x7FC00000u;
        }
        if (active) {
            const uint4 o = make_uint4(prmt32(V, Z, o0), prmt32(V, Z, o0 >> 16), prmt32(V, Z, o1),
                                       prmt32(V, Z, o1 >> 16));
            __stcs(reinterpret_cast<uint4*>(out + gi * G + p0), o);
            if (sub == 0) err_acc |= bad;
        }
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

// G >= 16: G/16 lanes per group, 16 weights per lane (two 16-byte stores).
// The lane's weights span four code bytes; their 20 selectors are packed into
// five words by PRMT and funnel-shifted to the lane's first weight, so the
// fixed per-lane work (loads, validation, scale) covers twice the weights.
// The selector table is held once per lane (word b * 32 + lane lies in bank
// `lane`), so a warp's 32 lookups of random bytes take one shared-memory
// wavefront instead of the 3-4 that bank conflicts on a single copy cost.
// 32 KB per CTA; six CTAs fit per SM (40 registers) and the grid is four
// such waves (the 72-matrix stack: 120 -> 117.5 us against one wave).
constexpr int kUnpackThreads = 256, kUnpackCtasPerSm = 6;

template <int G>
__global__ void __launch_bounds__(kUnpackThreads, kUnpackCtasPerSm) unpack16_kernel(
    const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales, int64_t num_groups,
    uint16_t* __restrict__ out, uint32_t* __restrict__ d_err) {
    constexpr int LPG = G / 16;
    constexpr int GPW = 32 / LPG;
    constexpr int B = bytes_per_group(G);
    constexpr int REAL = G - 5 * (B - 1);
    constexpr uint32_t PAD_SPAN = REAL == 1 ? 3u : (REAL == 2 ? 9u : (REAL == 3 ? 27u : 81u));
    constexpr uint32_t PAD_BASE = REAL == 1 ? 120u : (REAL == 2 ? 117u : (REAL == 3 ? 108u : 81u));
    // selectors of digits 0..3, one copy per lane; digit 4 = floor(b / 81) by arithmetic
    __shared__ uint32_t lut[256 * 32];
    fill_digit_selector_lut4_lanes(lut, threadIdx.x, blockDim.x);
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int sub = lane % LPG;
    const int p0 = 16 * sub;
    const int q_first = p0 / 5;  // weights p0..p0+15 lie in bytes q_first .. q_first+3
    const uint32_t shift = 8u * (uint32_t)(p0 - 5 * q_first);
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t stride = nwarps * GPW;
    uint32_t err_acc = 0;
    auto load = [&](int64_t base, uint32_t (&bv)[4], uint32_t& s) {
        const int64_t gi = base + lane / LPG;
        bv[0] = bv[1] = bv[2] = bv[3] = kZeroByte;
        s = 0;
        if (gi < num_groups) {
            const uint8_t* in = codes + gi * B;
#pragma unroll
            for (int t = 0; t < 4; ++t)
                if (q_first + t < B) bv[t] = __ldcs(in + q_first + t);
            s = __ldg(scales + gi);
        }
    };
    // code bytes and scale of the next two passes in flight
    uint32_t bv_next[4], s_next, bv_next2[4], s_next2;
    load(warp * GPW, bv_next, s_next);
    load(warp * GPW + stride, bv_next2, s_next2);
    for (int64_t base = warp * GPW; base < num_groups; base += stride) {
        const int64_t gi = base + lane / LPG;
        const bool active = gi < num_groups;
        const uint32_t bv[4] = {bv_next[0], bv_next[1], bv_next[2], bv_next[3]};
        const uint32_t s = s_next;
#pragma unroll
        for (int t = 0; t < 4; ++t) bv_next[t] = bv_next2[t];
        s_next = s_next2;
        load(base + 2 * stride, bv_next2, s_next2);
        uint32_t bad = scale_is_bad(s) ? TQ_DERR_SCALE : 0u;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint32_t b = bv[t];  // 121 (valid) past the group
            if (b >= 243) bad |= TQ_DERR_BYTE;
            else if (REAL < 5 && q_first + t == B - 1 && b - PAD_BASE >= PAD_SPAN) bad |= TQ_DERR_PADDING;
        }
        bad = seg_or_u32(bad, LPG);
        if (!active) bad = 0;
        // selector stream of the four bytes (5 per byte), then the lane's 16
        auto rec = [&](uint32_t b) { return make_uint2(lut[b * 32 + lane], 0x10u + 0x22u * ((b * 810u) >> 16)); };
        const uint2 e0 = rec(bv[0]), e1 = rec(bv[1]), e2 = rec(bv[2]), e3 = rec(bv[3]);
        const uint32_t W[5] = {e0.x, prmt32(e0.y, e1.x, 0x6540u), prmt32(prmt32(e1.x, e1.y, 0x0043u), e2.x, 0x5410u),
                               prmt32(prmt32(e2.x, e2.y, 0x0432u), e3.x, 0x4210u), prmt32(e3.x, e3.y, 0x4321u)};
        uint32_t V, Z;  // {-s, 0} and {+s, NaN}
        if (bad) {
            V = Z = 0x7FC07FC0u;
        } else {
            const uint32_t mag = (s == 0) ? 0u : scale_to_bf16_bits((uint16_t)s);
            V = mag ? (mag | 0x8000u) : 0u;
            Z = mag | 0x7FC00000u;
        }
        uint32_t v[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t o = __funnelshift_rc(W[j], W[j + 1], shift);
            v[2 * j] = prmt32(V, Z, o);
            v[2 * j + 1] = prmt32(V, Z, o >> 16);
        }
        if (active) {
            uint4* dst = reinterpret_cast<uint4*>(out + gi * G + p0);
            __stcs(dst, make_uint4(v[0], v[1], v[2], v[3]));
            __stcs(dst + 1, make_uint4(v[4], v[5], v[6], v[7]));
            if (sub == 0) err_acc |= bad;
        }
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

// Any G: one thread per group.
__global__ void __launch_bounds__(128) unpack_generic_kernel(
    const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales, int64_t num_groups,
    int G, uint16_t* __restrict__ out, uint32_t* __restrict__ d_err) {
    const int B = bytes_per_group(G);
    const int real = G - 5 * (B - 1);
    uint32_t err_acc = 0;
    for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < num_groups;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const uint8_t* in = codes + gi * B;
        const uint32_t s = scales[gi];
        uint32_t bad = scale_is_bad(s) ? TQ_DERR_SCALE : 0u;
        for (int q = 0; q < B; ++q) {
            const uint32_t p = byte_digit_pattern(in[q]);
            if (p & 0x8000u) bad |= TQ_DERR_BYTE;
            else if (q == B - 1 && (p & padding_mask(real)) != padding_ones(real)) bad |= TQ_DERR_PADDING;
        }
        const uint32_t mag = (s == 0) ? 0u : scale_to_bf16_bits((uint16_t)s);
        uint16_t* o = out + gi * G;
        for (int j = 0; j < G; ++j) {
            uint32_t v;
            if (bad) {
                v = kBf16NaN;
            } else {
                const uint32_t d = (byte_digit_pattern(in[j / 5]) >> (2 * (j % 5))) & 3u;
                v = (d == 1u || mag == 0u) ? 0u : (mag | (d == 0u ? 0x8000u : 0u));
            }
            o[j] = (uint16_t)v;
        }
        err_acc |= bad;
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

cudaError_t launch_unpack(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t K, int G,
                          uint16_t* out, uint32_t* d_err, cudaStream_t stream, int sm_count) {
    const int64_t num_groups = N * (K / G);
    if (num_groups == 0) return cudaSuccess;
    auto grid = [&](int64_t threads, int block) {
        int64_t b = (threads + block - 1) / block;
        const int64_t cap = (int64_t)sm_count * 16;
        return (int)(b > cap ? cap : (b < 1 ? 1 : b));
    };
#define TQ_UP_CASE(GG)                                                                          \
    case GG: {                                                                                  \
        const int64_t threads = (num_groups + (32 / (GG / 16)) - 1) / (32 / (GG / 16)) * 32;    \
        const int64_t blocks = (threads + kUnpackThreads - 1) / kUnpackThreads;                 \
        const int64_t cap = (int64_t)sm_count * kUnpackCtasPerSm * 4;                           \
        unpack16_kernel<GG><<<(int)(blocks < cap ? blocks : cap), kUnpackThreads, 0, stream>>>( \
            codes, scales, num_groups, out, d_err);                                             \
        return cudaGetLastError();                                                              \
    }
    switch (G) {
        case 8: {
            const int64_t threads = (num_groups + 3) / 4 * 32;
            unpack_pow2_kernel<8><<<grid(threads, 256), 256, 0, stream>>>(codes, scales, num_groups, out, d_err);
            return cudaGetLastError();
        }
        TQ_UP_CASE(16)
        TQ_UP_CASE(32)
        TQ_UP_CASE(64)
        TQ_UP_CASE(128)
        TQ_UP_CASE(256)
        default:
            break;
    }
#undef TQ_UP_CASE
    unpack_generic_kernel<<<grid(num_groups, 128), 128, 0, stream>>>(codes, scales, num_groups, G,
                                                                      out, d_err);
    return cudaGetLastError();
}

}  // namespace tq
