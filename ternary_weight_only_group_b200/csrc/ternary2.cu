// ternary2.cu -- the 2-bit ternary format: unpack to bf16 and the decode GEMV
// (CUDA cores, sm_100a).  The quantizer shares the group kernel of
// quantize_pack.cu (FMT = 2).
//
// Format ("Autoregressive Language Model on the 6502 Processor", summary:
// BitNet ternary weights, four parameters per byte): the groups, fp16 scales
// and trits of the base-3 codec ("precisit/pack-unpack-run", codec.py); code
// c = t + 1 in two bits, the first weight in the low bits, ceil(G/4) bytes
// per group, padding codes 1; code 3 is invalid.  With G % 16 == 0 a group is
// G/16 whole 32-bit words, which is what the word kernels below rely on.
//
// Decoding a word: byte i of the word holds weights 4i .. 4i+3.  Spreading
// the four 2-bit codes of a byte into the four bytes of a word (two
// multiply-and-mask steps) and mapping code c to the PRMT selector byte
// 0x10 + 0x22 c picks, per bf16 half, -s (c = 0), 0 (c = 1), +s (c = 2) or
// NaN (c = 3) from the pair V = {-s, 0}, Z = {+s, NaN}.  The GEMV skips the
// spreading: (c >> 2k) & 0x03030303 already holds the codes of weights k,
// k+4, k+8, k+12 in its four bytes, and the activations are staged in that
// order instead.
#include <atomic>

#include "tq_internal.cuh"

namespace tq {

namespace {

__device__ __forceinline__ void value_pair(uint32_t s, bool bad, uint32_t& V, uint32_t& Z) {
    if (bad) {
        V = Z = 0x7FC07FC0u;
    } else {
        const uint32_t mag = s == 0 ? 0u : scale_to_bf16_bits((uint16_t)s);
        V = mag ? (mag | 0x8000u) : 0u;  // {-s, 0}
        Z = mag | 0x7FC00000u;           // {+s, NaN}
    }
}

// Selector word of the four codes in byte x (0..255): code k in byte k.
__device__ __forceinline__ uint32_t spread_selectors(uint32_t x) {
    uint32_t u = (x * 0x1001u) & 0x000F000Fu;  // codes 0,1 in bits 0-3; codes 2,3 in bits 16-19
    u = (u * 0x41u) & 0x03030303u;             // code k in bits 8k, 8k+1
    return 0x10101010u + 0x22u * u;
}

// True if any 2-bit field of c is 3.
__device__ __forceinline__ bool has_code3(uint32_t c) { return (c & (c >> 1) & 0x55555555u) != 0; }

// ---------------------------------------------------------------- unpack

// G % 16 == 0, WPG = G/16 words per group: one lane per word (16 weights, two
// 16-byte stores).  A group's words sit in WPG consecutive lanes of a warp,
// which OR their error bits so a rejected group is NaN as a whole.
template <int WPG>
__global__ void __launch_bounds__(256) unpack2_words_kernel(const uint32_t* __restrict__ codes,
                                                            const uint16_t* __restrict__ scales, int64_t nwords,
                                                            uint16_t* __restrict__ out, uint32_t* __restrict__ d_err) {
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    uint32_t err_acc = 0;
    // the code words and scales of the next kPre passes are in flight (one
    // 4-byte word per lane and pass is too little to cover the load latency)
    constexpr int kPre = 4;
    auto load = [&](int64_t w, uint32_t& c, uint32_t& s) {
        c = 0x55555555u;  // past the end: zero trits, never stored
        s = 0;
        if (w < nwords) {
            c = __ldcs(codes + w);
            s = __ldg(scales + w / WPG);
        }
    };
    const int64_t first = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
    uint32_t cq[kPre], sq[kPre];
#pragma unroll
    for (int i = 0; i < kPre; ++i) load(first + i * stride + lane, cq[i], sq[i]);
    for (int64_t base = first; base < nwords; base += stride) {
        const int64_t w = base + lane;
        const bool active = w < nwords;
        const uint32_t c = cq[0], s = sq[0];
#pragma unroll
        for (int i = 0; i + 1 < kPre; ++i) {
            cq[i] = cq[i + 1];
            sq[i] = sq[i + 1];
        }
        load(base + kPre * stride + lane, cq[kPre - 1], sq[kPre - 1]);
        uint32_t bad = (scale_is_bad(s) ? TQ_DERR_SCALE : 0u) | (has_code3(c) ? TQ_DERR_BYTE : 0u);
        bad = seg_or_u32(bad, WPG);
        uint32_t V, Z;
        value_pair(s, bad != 0, V, Z);
        uint32_t v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t sel = spread_selectors((c >> (8 * i)) & 0xFFu);
            v[2 * i] = prmt32(V, Z, sel);
            v[2 * i + 1] = prmt32(V, Z, sel >> 16);
        }
        if (active) {
            uint4* dst = reinterpret_cast<uint4*>(out + w * 16);
            __stcs(dst, make_uint4(v[0], v[1], v[2], v[3]));
            __stcs(dst + 1, make_uint4(v[4], v[5], v[6], v[7]));
            if (lane % WPG == 0) err_acc |= bad;
        }
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

// Any G: one thread per group, byte loads, padding codes checked.
__global__ void __launch_bounds__(128) unpack2_generic_kernel(const uint8_t* __restrict__ codes,
                                                              const uint16_t* __restrict__ scales,
                                                              int64_t num_groups, int G, uint16_t* __restrict__ out,
                                                              uint32_t* __restrict__ d_err) {
    const int B = (G + 3) / 4;
    uint32_t err_acc = 0;
    for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < num_groups;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const uint8_t* in = codes + gi * B;
        const uint32_t s = scales[gi];
        uint32_t bad = scale_is_bad(s) ? TQ_DERR_SCALE : 0u;
        for (int q = 0; q < B; ++q) {
            const uint32_t b = in[q];
            if (has_code3(b)) bad |= TQ_DERR_BYTE;
            for (int i = 0; i < 4; ++i) {  // a padding code must be 1 (a 3 counts as an invalid code)
                const uint32_t f = (b >> (2 * i)) & 3u;
                if (4 * q + i >= G && f != 1u && f != 3u) bad |= TQ_DERR_PADDING;
            }
        }
        uint32_t V, Z;
        value_pair(s, bad != 0, V, Z);
        uint16_t* o = out + gi * G;
        for (int j = 0; j < G; ++j) {
            const uint32_t code = (in[j >> 2] >> (2 * (j & 3))) & 3u;
            o[j] = (uint16_t)prmt32(V, Z, 0x10u + 0x22u * code);
        }
        err_acc |= bad;
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

// ---------------------------------------------------------------- GEMV

constexpr int kG2Threads = 256;
constexpr int kG2Warps = kG2Threads / 32;
constexpr int kG2Unroll = 4;  // code words per lane in flight per row
constexpr size_t kG2MaxSmem = 96 * 1024;
template <int MT>
constexpr int kG2CtasPerSm = MT <= 2 ? 3 : 2;

// On entry every lane holds v[0..RB); on exit lane l < RB holds the sum over
// the warp of v[l] (halving exchanges, then a transposing butterfly).
template <int RB>
__device__ __forceinline__ float g2_transpose_reduce(float (&v)[RB]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o >= RB; o >>= 1) {
#pragma unroll
        for (int i = 0; i < RB; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
    }
#pragma unroll
    for (int n = RB / 2; n >= 1; n >>= 1) {
        const bool upper = (lane & n) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float keep = upper ? v[n + i] : v[i];
            const float send = upper ? v[i] : v[n + i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, n);
        }
    }
    return v[0];
}

__device__ __forceinline__ float fma_bf16_lo(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}

// Y[m][n] = sum_k X[m][k] * What[n][k], fp32 accumulation, MT <= 8 tokens,
// G = 16 * WPG.  A warp takes RB rows at a time; lane l reads code words l,
// l + 32, ... of each row (coalesced) and their scales.  The activations sit
// in shared memory per 16-column block b as two 16-byte halves in the order
// the selector words produce the weights: lo[b] = (x0,x4),(x8,x12),(x1,x5),
// (x9,x13); hi[b] = (x2,x6),(x10,x14),(x3,x7),(x11,x15).
template <int MT, int WPG>
__global__ void __launch_bounds__(kG2Threads, kG2CtasPerSm<MT>) gemv2_kernel(
    const uint16_t* __restrict__ X, int M, const uint32_t* __restrict__ codes, const uint16_t* __restrict__ scales,
    int64_t N, int K, void* __restrict__ Y, int y_bf16, uint32_t* __restrict__ d_err) {
    constexpr int RB = MT <= 2 ? 4 : 2;
    extern __shared__ __align__(16) uint4 xs[];  // [MT][2][K/16]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wpr = K / 16;  // code words per row
    const int ng = wpr / WPG;

    const int64_t nbatch = (N + RB - 1) / RB;
    const int64_t bt0 = (int64_t)blockIdx.x * kG2Warps + warp;  // this warp's first row batch
    // code words and scales of a row batch, words i0 + lane, i0 + 32 + lane, ...
    uint32_t cw[RB][kG2Unroll], sc[RB][kG2Unroll];
    auto load = [&](int64_t bt, int i0) {
        const int64_t n0 = bt * RB;
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int64_t n = n0 + r < N ? n0 + r : N - 1;  // rows past the end repeat the last, never stored
#pragma unroll
            for (int u = 0; u < kG2Unroll; ++u) {
                const int i = i0 + 32 * u + lane;
                cw[r][u] = 0x55555555u;
                sc[r][u] = 0u;
                if (i < wpr) {
                    cw[r][u] = __ldcs(codes + n * wpr + i);
                    sc[r][u] = __ldg(scales + n * ng + i / WPG);
                }
            }
        }
    };

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // Codes and scales are weights, not results of the preceding kernel: the
    // first batch's are requested before waiting for it (see tq2_gemv's
    // ordering rule); the activations only after.
    if (bt0 < nbatch) load(bt0, 0);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // stage the activations (written by the preceding kernel: L2 loads)
    for (int i = threadIdx.x; i < MT * wpr; i += kG2Threads) {
        const int m = i / wpr, b = i - m * wpr;
        uint4 a = make_uint4(0u, 0u, 0u, 0u), c = a;
        if (m < M) {
            const uint4* src = reinterpret_cast<const uint4*>(X + (int64_t)m * K + 16 * b);
            a = __ldcg(src);
            c = __ldcg(src + 1);
        }
        // a = X0..X3, c = X4..X7 with X_i = (x_2i, x_2i+1)
        xs[(2 * m) * wpr + b] = make_uint4(prmt32(a.x, a.z, 0x5410u), prmt32(c.x, c.z, 0x5410u),
                                           prmt32(a.x, a.z, 0x7632u), prmt32(c.x, c.z, 0x7632u));
        xs[(2 * m + 1) * wpr + b] = make_uint4(prmt32(a.y, a.w, 0x5410u), prmt32(c.y, c.w, 0x5410u),
                                               prmt32(a.y, a.w, 0x7632u), prmt32(c.y, c.w, 0x7632u));
    }
    __syncthreads();

    uint32_t err_acc = 0;
    for (int64_t bt = bt0; bt < nbatch; bt += (int64_t)gridDim.x * kG2Warps) {
        const int64_t n0 = bt * RB;
        float acc[MT][RB];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[m][r] = 0.f;
        for (int i0 = 0; i0 < wpr; i0 += 32 * kG2Unroll) {
            if (bt != bt0 || i0 != 0) load(bt, i0);
#pragma unroll
            for (int u = 0; u < kG2Unroll; ++u) {
                const int i = i0 + 32 * u + lane;
                if (i0 + 32 * u >= wpr) break;
                uint4 xl[MT], xh[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    xl[m] = make_uint4(0u, 0u, 0u, 0u);
                    xh[m] = xl[m];
                    if (i < wpr) {
                        xl[m] = xs[(2 * m) * wpr + i];
                        xh[m] = xs[(2 * m + 1) * wpr + i];
                    }
                }
#pragma unroll
                for (int r = 0; r < RB; ++r) {
                    const uint32_t c = cw[r][u], s = sc[r][u];
                    const bool bad = scale_is_bad(s) || has_code3(c);
                    if (bad && i < wpr) err_acc |= (scale_is_bad(s) ? TQ_DERR_SCALE : 0u) | (has_code3(c) ? TQ_DERR_BYTE : 0u);
                    uint32_t V, Z;
                    value_pair(s, bad, V, Z);
                    uint32_t wv[8];  // (w0,w4),(w8,w12),(w1,w5),(w9,w13),(w2,w6),(w10,w14),(w3,w7),(w11,w15)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t sel = 0x10101010u + 0x22u * ((c >> (2 * k)) & 0x03030303u);
                        wv[2 * k] = prmt32(V, Z, sel);
                        wv[2 * k + 1] = prmt32(V, Z, sel >> 16);
                    }
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const uint32_t xv[8] = {xl[m].x, xl[m].y, xl[m].z, xl[m].w, xh[m].x, xh[m].y, xh[m].z, xh[m].w};
                        float a = acc[m][r];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            a = fma_bf16_lo(wv[k], xv[k], a);
                            a = fma_bf16_hi(wv[k], xv[k], a);
                        }
                        acc[m][r] = a;
                    }
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float tot = g2_transpose_reduce<RB>(acc[m]);
            if (lane < RB && m < M && n0 + lane < N) {
                const int64_t o = (int64_t)m * N + n0 + lane;
                if (y_bf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(tot);
                else reinterpret_cast<float*>(Y)[o] = tot;
            }
        }
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

template <int MT, int WPG>
cudaError_t launch_gemv2_t(const uint16_t* X, int M, const uint32_t* codes, const uint16_t* scales, int64_t N, int K,
                           void* Y, int y_bf16, uint32_t* d_err, cudaStream_t stream, int sm_count) {
    auto kern = gemv2_kernel<MT, WPG>;
    const size_t smem = (size_t)MT * K * 2;
    static SmemAttr smem_attr;
    if ((int)smem > 48 * 1024)
        if (cudaError_t e = smem_attr.ensure(kern, (int)smem)) return e;
    constexpr int RB = MT <= 2 ? 4 : 2;
    const int64_t nbatch = (N + RB - 1) / RB;
    const int64_t want = (nbatch + kG2Warps - 1) / kG2Warps;
    const int64_t cap = (int64_t)sm_count * kG2CtasPerSm<MT>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < cap ? want : cap));
    cfg.blockDim = dim3(kG2Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, X, M, codes, scales, N, K, Y, y_bf16, d_err);
}

template <int WPG>
cudaError_t launch_gemv2_w(const uint16_t* X, int M, const uint32_t* codes, const uint16_t* scales, int64_t N, int K,
                           void* Y, int y_bf16, uint32_t* d_err, cudaStream_t stream, int sm_count) {
    if (M == 1) return launch_gemv2_t<1, WPG>(X, M, codes, scales, N, K, Y, y_bf16, d_err, stream, sm_count);
    if (M == 2) return launch_gemv2_t<2, WPG>(X, M, codes, scales, N, K, Y, y_bf16, d_err, stream, sm_count);
    if (M <= 4) return launch_gemv2_t<4, WPG>(X, M, codes, scales, N, K, Y, y_bf16, d_err, stream, sm_count);
    return launch_gemv2_t<8, WPG>(X, M, codes, scales, N, K, Y, y_bf16, d_err, stream, sm_count);
}

}  // namespace

cudaError_t launch_unpack2(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t K, int G, uint16_t* out,
                           uint32_t* d_err, cudaStream_t stream, int sm_count) {
    const int64_t num_groups = N * (K / G);
    if (num_groups == 0) return cudaSuccess;
    // up to 32 CTAs per SM, four waves of the eight that fit: each thread
    // walks fewer passes (the 72-matrix stack at G = 64 / 128: 134 / 129 us
    // with 8 per SM, 123 / 119 us with 32, 161 us with one CTA per 256 words)
    const int64_t cap = (int64_t)sm_count * 32;
    if (G % 16 == 0 && G <= 256 && (G & (G - 1)) == 0) {
        const int64_t nwords = N * K / 16;
        const int64_t blocks = (nwords + 255) / 256;
        const int grid = (int)(blocks < cap ? blocks : cap);
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes);
        switch (G / 16) {
            case 1: unpack2_words_kernel<1><<<grid, 256, 0, stream>>>(cw, scales, nwords, out, d_err); break;
            case 2: unpack2_words_kernel<2><<<grid, 256, 0, stream>>>(cw, scales, nwords, out, d_err); break;
            case 4: unpack2_words_kernel<4><<<grid, 256, 0, stream>>>(cw, scales, nwords, out, d_err); break;
            case 8: unpack2_words_kernel<8><<<grid, 256, 0, stream>>>(cw, scales, nwords, out, d_err); break;
            default: unpack2_words_kernel<16><<<grid, 256, 0, stream>>>(cw, scales, nwords, out, d_err); break;
        }
        return cudaGetLastError();
    }
    const int64_t blocks = (num_groups + 127) / 128;
    unpack2_generic_kernel<<<(int)(blocks < cap ? blocks : cap), 128, 0, stream>>>(codes, scales, num_groups, G, out,
                                                                                  d_err);
    return cudaGetLastError();
}

// Returns cudaErrorNotSupported for shapes the kernel does not cover (G not
// in {16, 32, 64, 128, 256}, or K too large for the staged activations).
cudaError_t launch_gemv2(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales, int64_t N,
                         int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err, cudaStream_t stream, int sm_count) {
    if (G % 16 != 0 || G > 256 || (G & (G - 1)) != 0) return cudaErrorNotSupported;
    if (K > (int64_t)(kG2MaxSmem / 2)) return cudaErrorNotSupported;
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes);
    const size_t osz = y_bf16 ? 2 : 4;
    for (int64_t m0 = 0; m0 < M;) {
        // tokens per launch: up to 8, as many as the shared-memory budget allows
        int mt = (int)(M - m0 < 8 ? M - m0 : 8);
        while (mt > 1 && (size_t)(mt <= 2 ? mt : (mt <= 4 ? 4 : 8)) * K * 2 > kG2MaxSmem) mt = mt <= 2 ? 1 : (mt <= 4 ? 2 : 4);
        const uint16_t* Xm = X + m0 * K;
        void* Ym = static_cast<char*>(Y) + (size_t)m0 * N * osz;
        cudaError_t e;
        switch (G / 16) {
            case 1: e = launch_gemv2_w<1>(Xm, mt, cw, scales, N, (int)K, Ym, y_bf16, d_err, stream, sm_count); break;
            case 2: e = launch_gemv2_w<2>(Xm, mt, cw, scales, N, (int)K, Ym, y_bf16, d_err, stream, sm_count); break;
            case 4: e = launch_gemv2_w<4>(Xm, mt, cw, scales, N, (int)K, Ym, y_bf16, d_err, stream, sm_count); break;
            case 8: e = launch_gemv2_w<8>(Xm, mt, cw, scales, N, (int)K, Ym, y_bf16, d_err, stream, sm_count); break;
            default: e = launch_gemv2_w<16>(Xm, mt, cw, scales, N, (int)K, Ym, y_bf16, d_err, stream, sm_count); break;
        }
        if (e != cudaSuccess) return e;
        m0 += mt;
    }
    return cudaSuccess;
}

}  // namespace tq
