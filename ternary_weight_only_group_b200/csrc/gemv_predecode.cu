// gemv_predecode.cu -- decode GEMV for small matrices, weights decoded before
// the activations are waited for (CUDA cores, sm_100a).
//
// Y[n] = sum_k X[k] * What[n][k] with What = t * RNE_bf16(scale) (tiny-llm
// "Week 2 Day 3: Quantize the Model", "Mathematical Formulation"; the
// decoding of "precisit/pack-unpack-run", codec.py), fp32 accumulation,
// 1 <= M <= 8 tokens.
//
// In a chain of dependent layers a kernel's weights are known long before its
// activations.  Each CTA (one per SM, R rows) therefore stages its codes and
// scales in shared memory with one round of cp.async and decodes them to bf16
// BEFORE griddepcontrol.wait, while the previous kernels are still running
// (up to three CTAs share an SM, so two later launches decode while one
// computes).  After the wait only the activation load, one mixed-precision
// FMA per weight and token (bf16 inputs, fp32 accumulator), a transposing
// butterfly per eight rows and token and the stores remain: no tables, no
// cluster barrier.  When one CTA per SM would need more shared memory than
// fits, two CTAs per SM take half the rows each (less overlap).
//
// Decode: one lane per 64 weights of a group (a whole group when G <= 64).
// Code byte i of the lane's window contributes its five PRMT selector bytes
// (digit d -> 0x10 + 0x22 d, picking -s, 0, +s or NaN) at stream byte 5i,
// which is byte (i mod 4) of word (5i) div 4; four 256-entry tables hold every
// byte's selectors pre-shifted by 0..3 bytes, so the stream is built by ORs.
// An invalid byte (>= 243) selects NaN for its digits, a rejected scale or a
// padding digit other than 1 makes the lane's weights NaN; either way the
// row's output is NaN, and the error bits are recovered by rescanning the
// NaN rows at the end.
//
// Covers G = 8 * 2^k (8 <= G <= 256), K % 512 == 0, and matrices whose
// per-CTA rows fit in about 100 KB of bf16; the lookup-table GEMV takes the
// rest.
#include <atomic>
#include <type_traits>

#include "tq_internal.cuh"

namespace tq {

constexpr int kPdThreads = 256;
constexpr int kPdWarps = kPdThreads / 32;
constexpr size_t kPdMaxSmem = 110 * 1024;  // at least two CTAs per SM
constexpr int kPdTableBytes = 4 * 256 * 8;

// The four shifted selector tables: entry [o][b] is the 40-bit selector
// record of byte b shifted left by 8 o bits, as (low word, high word).
struct __align__(16) PdSelectorTables {
    uint2 t[4][256];
    constexpr PdSelectorTables() : t{} {
        for (int b = 0; b < 256; ++b) {
            unsigned long long rec = 0;
            uint32_t v = (uint32_t)b;
            for (int i = 0; i < 5; ++i) {
                const uint32_t d = b >= 243 ? 3u : v % 3u;
                v /= 3u;
                rec |= (unsigned long long)(0x10u + 0x22u * d) << (8 * i);
            }
            for (int o = 0; o < 4; ++o) {
                const unsigned long long sh = rec << (8 * o);
                t[o][b].x = (uint32_t)sh;
                t[o][b].y = (uint32_t)(sh >> 32);
            }
        }
    }
};
__device__ const PdSelectorTables kPdSelectors;

// Bytes reserved for a staged range of n bytes: its offset within a 16-byte
// chunk (< 16) plus the range, rounded to 16.
__host__ __device__ constexpr int pd_codes_area(int n) { return (n + 16 + 15) & ~15; }

// Shared memory: [selector tables, later the MT x K activations] | R x K
// decoded bf16 (swizzled chunks) | staged codes | staged scales.
__host__ __device__ constexpr int pd_head_bytes(int K, int MT) {
    return MT * K * 2 > kPdTableBytes ? MT * K * 2 : kPdTableBytes;
}

template <int RB>
__device__ __forceinline__ float pd_transpose_reduce(float (&v)[RB]) {
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

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src_global) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst_smem)),
                 "l"(__cvta_generic_to_global(src_global))
                 : "memory");
}

// Copies src[0, nbytes) into shared memory at dst + (src & 15), so that the
// 16-byte chunks of the source land on 16-byte boundaries: whole chunks by
// cp.async (all in flight at once), the ragged head and tail by byte loads.
// Nothing outside [src, src + nbytes) is read.  The caller commits, waits
// with cp.async.wait_all and a barrier.
__device__ __forceinline__ const unsigned char* stage_bytes(unsigned char* dst, const unsigned char* src,
                                                            int nbytes, int tid, int nthreads) {
    const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), s1 = s0 + (uintptr_t)nbytes;
    const uintptr_t a0 = s0 & ~(uintptr_t)15;
    const uintptr_t m0 = (s0 + 15) & ~(uintptr_t)15, m1 = s1 & ~(uintptr_t)15;
    if (m0 >= m1) {  // no whole chunk: bytes only
        for (int i = tid; i < nbytes; i += nthreads) dst[s0 - a0 + i] = src[i];
    } else {
        if (tid < 16 && s0 + tid < m0) dst[s0 - a0 + tid] = src[tid];
        const int j = tid - 16;
        if (j >= 0 && j < 16 && m1 + j < s1) dst[m1 - a0 + j] = src[m1 - s0 + j];
        const int nchunks = (int)((m1 - m0) >> 4);
        for (int i = tid; i < nchunks; i += nthreads)
            cp_async16(dst + (m0 - a0) + 16 * (size_t)i, reinterpret_cast<const void*>(m0 + 16 * (uintptr_t)i));
    }
    return dst + (s0 - a0);
}

__device__ __forceinline__ void store_y(void* Y, int y_bf16, int64_t n, float v) {
    if (y_bf16) reinterpret_cast<__nv_bfloat16*>(Y)[n] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(Y)[n] = v;
}

// d = a * b + c with bf16 a, b and an fp32 c, rounded once to fp32: the same
// value as fmaf on the widened inputs (the widening is exact).
__device__ __forceinline__ float fma_bf16(uint16_t a, uint16_t b, float c) {
    float d;
    asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
    return d;
}

// The 16-byte chunk c (columns 8c .. 8c+7) of a decoded row sits at chunk
// c ^ ((c >> 3) & 7): a permutation inside each aligned run of 8 chunks.
// With K % 512 == 0 a row holds a multiple of 64 chunks, so the same formula
// applied to the chunk index counted from the first row gives the same place.
// Decode lanes write chunks G / 8 apart and the FMA lanes read consecutive
// chunks; both are free of bank conflicts this way.
__device__ __forceinline__ int pd_swizzle(int c) { return c ^ ((c >> 3) & 7); }

// Code bytes per group: base-3 (FMT 3) ceil(G/5) + 2 ... as the codec
// defines; 2-bit (FMT 2, G a multiple of 16) G/4.
template <int G, int FMT>
__host__ __device__ constexpr int pd_group_bytes() { return FMT == 3 ? bytes_per_group(G) : G / 4; }

// The 2-bit format's decode of one lane's 16 * NWD weights: word q of the
// lane's codes holds columns 16 q .. 16 q + 15 (code c = t + 1 of column j
// in bits 2 (j mod 4) of byte j / 4); (w >> 2k) & 0x03030303 holds the codes
// of columns k, k+4, k+8, k+12, mapped to the selector bytes 0x10 + 0x22 c
// of {V, Z} and interleaved by PRMT into the selector pairs of adjacent
// columns (code 3 selects NaN).  `put(k, v)` gets chunk k (columns 8k ..
// 8k+7) as four bf16 pairs.
template <int NWD, class Put>
__device__ __forceinline__ void pd_decode_2bit(const uint32_t (&wd)[NWD], uint32_t V, uint32_t Z, Put&& put) {
#pragma unroll
    for (int q = 0; q < NWD; ++q) {
        uint32_t sel[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) sel[k] = 0x10101010u + 0x22u * ((wd[q] >> (2 * k)) & 0x03030303u);
        const uint32_t p01a = prmt32(sel[0], sel[1], 0x5140u);  // columns (0,1) low half, (4,5) high half
        const uint32_t p23a = prmt32(sel[2], sel[3], 0x5140u);  // (2,3), (6,7)
        const uint32_t p01b = prmt32(sel[0], sel[1], 0x7362u);  // (8,9), (12,13)
        const uint32_t p23b = prmt32(sel[2], sel[3], 0x7362u);  // (10,11), (14,15)
        put(2 * q, make_uint4(prmt32(V, Z, p01a), prmt32(V, Z, p23a), prmt32(V, Z, p01a >> 16),
                              prmt32(V, Z, p23a >> 16)));
        put(2 * q + 1, make_uint4(prmt32(V, Z, p01b), prmt32(V, Z, p23b), prmt32(V, Z, p01b >> 16),
                                  prmt32(V, Z, p23b >> 16)));
    }
}

template <int G, int MT, int FMT>
__global__ void __launch_bounds__(kPdThreads, MT == 1 ? 3 : 2) gemv_predecode_kernel(
    const uint16_t* __restrict__ X, int M, const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
    int64_t N, int K, int R, void* __restrict__ Y, int y_bf16, uint32_t* __restrict__ d_err) {
    static_assert(FMT == 3 || G % 16 == 0, "2-bit lanes decode whole 32-bit code words");
    constexpr int B = pd_group_bytes<G, FMT>();
    constexpr int REAL = G - 5 * (B - 1);   // real digits in a group's last byte
    constexpr int SW = G < 64 ? G : 64;     // weights a decode lane writes
    constexpr int LPG = G / SW;             // lanes per group
    constexpr int NBY = LPG == 1 ? B : 14;  // code bytes in the lane's window
    constexpr int NW = (5 * NBY + 3) / 4 + 1;
    constexpr int NCH = SW / 8;             // 16-byte chunks a lane writes
    // A canonical last byte has digits REAL..4 equal to 1, i.e. it lies in
    // [PAD_BASE, PAD_BASE + 3^REAL) with PAD_BASE = sum_{i=REAL}^{4} 3^i.
    constexpr uint32_t PAD_SPAN = REAL == 1 ? 3u : (REAL == 2 ? 9u : (REAL == 3 ? 27u : 81u));
    constexpr uint32_t PAD_BASE = REAL == 1 ? 120u : (REAL == 2 ? 117u : (REAL == 3 ? 108u : 81u));

    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float red[kPdWarps * 8 * MT];  // slice sums when the chunks are split over warps
    const uint2* tabs = reinterpret_cast<const uint2*>(smem);  // [4][256]
    uint16_t* w = reinterpret_cast<uint16_t*>(smem + pd_head_bytes(K, MT));  // [R][K] decoded bf16

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row0 = (int64_t)blockIdx.x * R;
    const int nrows = (int)(N - row0 < (int64_t)R ? N - row0 : (int64_t)R);
    const int ng = K / G;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // ---- stage the selector tables and this CTA's codes and scales (its rows
    // are contiguous) in one round of copies
    const int ngroups = nrows * ng;
    unsigned char* raw = smem + pd_head_bytes(K, MT) + (size_t)R * K * 2;
    if (FMT == 3)
        for (int i = threadIdx.x; i < kPdTableBytes / 16; i += kPdThreads)
            cp_async16(smem + 16 * i, reinterpret_cast<const unsigned char*>(&kPdSelectors) + 16 * i);
    const unsigned char* craw = stage_bytes(raw, codes + row0 * ng * B, ngroups * B, threadIdx.x, kPdThreads);
    const uint16_t* sraw = reinterpret_cast<const uint16_t*>(
        stage_bytes(raw + pd_codes_area(R * ng * B), reinterpret_cast<const unsigned char*>(scales + row0 * ng),
                    ngroups * 2, threadIdx.x, kPdThreads));
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();

    // ---- decode (weights only: no dependence on earlier kernels)
    if constexpr (FMT == 2) {
        constexpr int NWD = SW / 16;  // code words of a lane
        for (int u = threadIdx.x; u < ngroups * LPG; u += kPdThreads) {
            const int gl = u / LPG, sub = u - gl * LPG;
            const uint32_t s = sraw[gl];
            // the staged copy keeps the source's offset within 16 bytes, and
            // codes, rows and groups are 4-byte aligned: whole words
            const uint32_t* in = reinterpret_cast<const uint32_t*>(craw + (size_t)gl * B + (size_t)sub * (SW / 4));
            uint32_t wd[NWD];
#pragma unroll
            for (int i = 0; i < NWD; ++i) wd[i] = in[i];
            uint32_t V, Z;  // {-s, 0} and {+s, NaN}
            if (scale_is_bad(s)) {
                V = Z = 0x7FC07FC0u;
            } else {
                const uint32_t mag = (s == 0) ? 0u : scale_to_bf16_bits((uint16_t)s);
                V = mag ? (mag | 0x8000u) : 0u;
                Z = mag | 0x7FC00000u;
            }
            const int cg0 = u * NCH;
            pd_decode_2bit<NWD>(wd, V, Z,
                                [&](int k, uint4 v) { *reinterpret_cast<uint4*>(w + 8 * pd_swizzle(cg0 + k)) = v; });
        }
    } else
    for (int u = threadIdx.x; u < ngroups * LPG; u += kPdThreads) {
        const int gl = u / LPG, sub = u - gl * LPG;  // group inside the CTA, lane's part of it
        const int p0 = SW * sub;                     // first weight of the part
        const int q_first = p0 / 5;
        const uint32_t s = sraw[gl];
        const unsigned char* in = craw + (size_t)gl * B + q_first;
        uint32_t Wd[NW];
#pragma unroll
        for (int i = 0; i < NW; ++i) Wd[i] = 0u;
#pragma unroll
        for (int i = 0; i < NBY; ++i) {
            const uint2 e = tabs[(i & 3) * 256 + in[i]];
            Wd[(5 * i) / 4] |= e.x;
            Wd[(5 * i) / 4 + 1] |= e.y;
        }
        bool bad = scale_is_bad(s);
        if (REAL < 5 && sub == LPG - 1)  // this part holds the group's last byte
            bad |= (uint32_t)craw[(size_t)gl * B + B - 1] - PAD_BASE >= PAD_SPAN;
        uint32_t V, Z;  // {-s, 0} and {+s, NaN}
        if (bad) {
            V = Z = 0x7FC07FC0u;
        } else {
            const uint32_t mag = (s == 0) ? 0u : scale_to_bf16_bits((uint16_t)s);
            V = mag ? (mag | 0x8000u) : 0u;
            Z = mag | 0x7FC00000u;
        }
        const uint32_t shift = 8u * (uint32_t)(p0 - 5 * q_first);  // 0 whenever LPG == 1
        const int cg0 = u * NCH;  // first chunk, counted from the CTA's first row
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
            uint32_t o0, o1;
            if (LPG == 1) {
                o0 = Wd[2 * k];
                o1 = Wd[2 * k + 1];
            } else {
                o0 = __funnelshift_rc(Wd[2 * k], Wd[2 * k + 1], shift);
                o1 = __funnelshift_rc(Wd[2 * k + 1], Wd[2 * k + 2], shift);
            }
            *reinterpret_cast<uint4*>(w + 8 * pd_swizzle(cg0 + k)) =
                make_uint4(prmt32(V, Z, o0), prmt32(V, Z, o0 >> 16), prmt32(V, Z, o1), prmt32(V, Z, o1 >> 16));
        }
    }

    // ---- activations come from the previous kernel: one round of L2 loads
    // (not through L1, which may hold lines of an earlier kernel that shared
    // the SM) into the space of the selector tables, which are no longer used.
    const int nchunk = K / 8;  // 8-column chunks
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint4* xs = reinterpret_cast<uint4*>(smem);  // [MT][nchunk]; tokens past M are zero
    for (int c0 = 0; c0 < MT * nchunk; c0 += 4 * kPdThreads) {
        uint4 xv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + threadIdx.x + j * kPdThreads;
            xv[j] = make_uint4(0u, 0u, 0u, 0u);
            if (c < M * nchunk) xv[j] = __ldcg(reinterpret_cast<const uint4*>(X) + c);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + threadIdx.x + j * kPdThreads;
            if (c < MT * nchunk) xs[c] = xv[j];
        }
    }
    __syncthreads();

    // ---- work units: (batch of RB rows, slice of the chunks); with fewer
    // than eight batches the chunks are split over the idle warps and the
    // slices' sums meet in shared memory.  RB = 4 rows for one token (the
    // FFN projections' 7..25 rows per CTA then keep most warps busy without
    // the cross-warp combine: 3.3 -> 3.1 us per launch in the decode chain),
    // 8 rows up to 4 tokens, 4 rows for 8 tokens (the accumulators stay at 32
    // per lane).
    constexpr int RB = MT == 1 ? 4 : (MT <= 4 ? 8 : 4);
    const int nb = (nrows + RB - 1) / RB;
    const int ks = nb >= kPdWarps ? 1 : kPdWarps / nb;
    uint32_t err_acc = 0;
    for (int u = warp; u < nb * ks; u += kPdWarps) {
        const int b = u / ks, sl = u - b * ks;
        const int rb0 = RB * b;
        int roff[RB];  // element offset of each row (rows past the end repeat the last, never stored)
#pragma unroll
        for (int i = 0; i < RB; ++i) roff[i] = min(rb0 + i, nrows - 1) * K;
        float acc[MT][RB];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int i = 0; i < RB; ++i) acc[m][i] = 0.f;
#pragma unroll 2
        for (int c = lane + 32 * sl; c < nchunk; c += 32 * ks) {
            uint32_t xx[MT][4];
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const uint4 xv = xs[m * nchunk + c];
                xx[m][0] = xv.x;
                xx[m][1] = xv.y;
                xx[m][2] = xv.z;
                xx[m][3] = xv.w;
            }
            const int pc8 = 8 * pd_swizzle(c);
#pragma unroll
            for (int i = 0; i < RB; ++i) {
                const uint4 wv = *reinterpret_cast<const uint4*>(w + roff[i] + pc8);
                const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        acc[m][i] = fma_bf16((uint16_t)ww[h], (uint16_t)xx[m][h], acc[m][i]);
                        acc[m][i] = fma_bf16((uint16_t)(ww[h] >> 16), (uint16_t)(xx[m][h] >> 16), acc[m][i]);
                    }
                }
            }
        }
        float tot[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) tot[m] = pd_transpose_reduce<RB>(acc[m]);
        if (lane < RB) {
            const int rr = rb0 + lane;
            if (ks == 1) {
                if (rr < nrows) {
                    if (tot[0] != tot[0])
                        err_acc |= FMT == 3 ? scan_row_errors(codes + (row0 + rr) * ng * B, scales + (row0 + rr) * ng, ng, G, B)
                                            : scan_row_errors2(codes + (row0 + rr) * ng * B, scales + (row0 + rr) * ng, ng, G);
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m < M) store_y(Y, y_bf16, (int64_t)m * N + row0 + rr, tot[m]);
                }
            } else {
#pragma unroll
                for (int m = 0; m < MT; ++m) red[(sl * (RB * nb) + rr) * MT + m] = tot[m];  // ks * RB * nb <= 64
            }
        }
    }
    if (ks > 1) {  // uniform across the CTA
        __syncthreads();
        const int rr = threadIdx.x;
        if (rr < nrows) {
            float tot[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) tot[m] = 0.f;
            for (int sl = 0; sl < ks; ++sl)
#pragma unroll
                for (int m = 0; m < MT; ++m) tot[m] += red[(sl * (RB * nb) + rr) * MT + m];
            if (tot[0] != tot[0])
                err_acc |= FMT == 3 ? scan_row_errors(codes + (row0 + rr) * ng * B, scales + (row0 + rr) * ng, ng, G, B)
                                    : scan_row_errors2(codes + (row0 + rr) * ng * B, scales + (row0 + rr) * ng, ng, G);
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M) store_y(Y, y_bf16, (int64_t)m * N + row0 + rr, tot[m]);
        }
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

template <int G, int MT, int FMT>
static cudaError_t launch_pd(const uint16_t* X, int M, const uint8_t* codes, const uint16_t* scales, int64_t N,
                             int K, int R, int grid, size_t smem, void* Y, int y_bf16, uint32_t* d_err,
                             cudaStream_t stream) {
    auto kern = gemv_predecode_kernel<G, MT, FMT>;
    static SmemAttr smem_attr;
    if (cudaError_t e = smem_attr.ensure(kern, (int)smem)) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kPdThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, X, M, codes, scales, N, K, R, Y, y_bf16, d_err);
}

template <int MT, int FMT>
static cudaError_t launch_pd_g(int G, const uint16_t* X, int M, const uint8_t* codes, const uint16_t* scales,
                               int64_t N, int K, int R, int grid, size_t smem, void* Y, int y_bf16, uint32_t* d_err,
                               cudaStream_t stream) {
    switch (G) {
        case 8:
            if constexpr (FMT == 3) return launch_pd<8, MT, 3>(X, M, codes, scales, N, K, R, grid, smem, Y, y_bf16, d_err, stream);
            else return cudaErrorNotSupported;
        case 16: return launch_pd<16, MT, FMT>(X, M, codes, scales, N, K, R, grid, smem, Y, y_bf16, d_err, stream);
        case 32: return launch_pd<32, MT, FMT>(X, M, codes, scales, N, K, R, grid, smem, Y, y_bf16, d_err, stream);
        case 64: return launch_pd<64, MT, FMT>(X, M, codes, scales, N, K, R, grid, smem, Y, y_bf16, d_err, stream);
        case 128: return launch_pd<128, MT, FMT>(X, M, codes, scales, N, K, R, grid, smem, Y, y_bf16, d_err, stream);
        default: return launch_pd<256, MT, FMT>(X, M, codes, scales, N, K, R, grid, smem, Y, y_bf16, d_err, stream);
    }
}

// Returns cudaErrorNotSupported when the shape is not covered.
cudaError_t launch_gemv_predecode(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                                  int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                                  cudaStream_t stream, int sm_count, int fmt) {
    if (M < 1 || M > 8 || K % 512 != 0 || N < 1 || K > 65536) return cudaErrorNotSupported;
    if (G != 8 && G != 16 && G != 32 && G != 64 && G != 128 && G != 256) return cudaErrorNotSupported;
    if (fmt != 3 && (fmt != 2 || G % 16 != 0 || (reinterpret_cast<uintptr_t>(codes) & 3))) return cudaErrorNotSupported;
    const int MT = M == 1 ? 1 : (M == 2 ? 2 : (M <= 4 ? 4 : 8));
    const int64_t ng = K / G, B = fmt == 3 ? bytes_per_group(G) : G / 4;
    // one CTA per SM if it fits (later launches then decode beside it), else two
    for (int per_sm = 1; per_sm <= 2; ++per_sm) {
        const int64_t R = (N + (int64_t)sm_count * per_sm - 1) / ((int64_t)sm_count * per_sm);
        if (R * K * 2 > (int64_t)kPdMaxSmem) continue;
        const size_t smem = (size_t)pd_head_bytes((int)K, MT) + (size_t)(R * K * 2) +
                            (size_t)pd_codes_area((int)(R * ng * B)) + (size_t)pd_codes_area((int)(R * ng * 2));
        if (smem > kPdMaxSmem) continue;
        const int grid = (int)((N + R - 1) / R);
        auto go = [&](auto fmt_tag) {
            constexpr int F = decltype(fmt_tag)::value;
            if (MT == 1) return launch_pd_g<1, F>(G, X, (int)M, codes, scales, N, (int)K, (int)R, grid, smem, Y, y_bf16, d_err, stream);
            if (MT == 2) return launch_pd_g<2, F>(G, X, (int)M, codes, scales, N, (int)K, (int)R, grid, smem, Y, y_bf16, d_err, stream);
            if (MT == 4) return launch_pd_g<4, F>(G, X, (int)M, codes, scales, N, (int)K, (int)R, grid, smem, Y, y_bf16, d_err, stream);
            return launch_pd_g<8, F>(G, X, (int)M, codes, scales, N, (int)K, (int)R, grid, smem, Y, y_bf16, d_err, stream);
        };
        return fmt == 3 ? go(std::integral_constant<int, 3>{}) : go(std::integral_constant<int, 2>{});
    }
    return cudaErrorNotSupported;
}

}  // namespace tq
