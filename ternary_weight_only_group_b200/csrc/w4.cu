// w4.cu -- the W4A16 affine format: decode GEMV on the CUDA cores (sm_100a).
//
// Format (tiny-llm "Week 2 Day 3: Quantize the Model", "Group-Wise Affine
// Quantization", "Reconstruct a Stored Group", "Packed Storage Layout"):
// unsigned 4-bit codes q, eight per 32-bit word with the first code in the
// low nibble, and per group of G columns a signed bf16 scale s and a bf16
// bias b; the weight is w = q * s + b.
//
// Matmul ("Mathematical Formulation", "Computation Flow"; the bias factored
// out of the group's dot product as in "Stage 2: SIMD Matvec"):
//   Y[m][n] = sum_g ( s[n,g] * sum_{j in g} q[n,j] X[m,j] + b[n,g] * sum_{j in g} X[m,j] ),
// fp32 accumulation; the group sums of X are formed once per launch.
//
// Kernel (G a multiple of 32, K a multiple of 32, up to 8 tokens per
// launch): a warp takes one row at a time; lane l owns the 32-column chunks
// l, l + 32, ... of the row (one 16-byte code load each, the chunk inside one
// group).  Codes become exact fp32 integers with one PRMT per weight (the
// nibble placed in the mantissa of 2^23, then 2^23 subtracted by a paired
// fp32 add) and meet the activations in paired fp32 FMAs (fma.rn.f32x2).  The
// activations sit in shared memory as fp32, each chunk's eight float4 pieces
// rotated by the chunk index so that a warp's loads never conflict.  Code
// words are requested several rows ahead; the per-row lane partials of eight
// rows are summed by a transposing butterfly.  Codes, scales and biases do
// not depend on earlier kernels: the first rows' loads are issued before
// griddepcontrol.wait, the activations are read after it.  Other shapes take
// a plain one-warp-per-row kernel.
#include <cstdio>
#include <cstdlib>

#include "tq_internal.cuh"

namespace tq {

namespace {

constexpr int kW4Threads = 256;
constexpr int kW4Warps = kW4Threads / 32;

struct W4Args {
    const uint16_t* X;
    int M, m0;           // tokens of this launch: rows m0 .. m0 + M - 1 of X
    const uint4* codes;  // [N][K/32] 16-byte chunks
    const uint16_t* scales;
    const uint16_t* biases;
    int64_t N;
    int K, G, ng, nchunk;
    void* Y;
    int y_bf16;
};

__device__ __forceinline__ float bf16f(uint32_t h) { return __uint_as_float(h << 16); }

// Transposing butterfly over a warp: lane l (l < RB) ends with the warp sum of v[l].
template <int RB>
__device__ __forceinline__ float w4_reduce(float (&v)[RB], int lane) {
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

// Rows per warp batch (one butterfly) and rows of code loads in flight, by
// tokens and chunks per lane: more tokens keep fewer rows in registers.
template <int MT>
__host__ __device__ constexpr int w4_rb() { return MT <= 2 ? 8 : (MT == 4 ? 4 : 2); }
template <int MT, int CPL>
__host__ __device__ constexpr int w4_depth() {
    return (MT == 1 ? 8 : 4) / CPL < 1 ? 1 : ((MT == 1 ? 8 : 4) / CPL > w4_rb<MT>() ? w4_rb<MT>() : (MT == 1 ? 8 : 4) / CPL);
}

// MT tokens (1, 2, 4, 8), CPL chunks per lane and row at most (K <= 1024 CPL).
template <int MT, int CPL>
__global__ void __launch_bounds__(kW4Threads, MT <= 2 ? 2 : 1) gemv_w4_kernel(const W4Args a) {
    constexpr int RB = w4_rb<MT>();        // rows per warp batch
    constexpr int D = w4_depth<MT, CPL>();  // rows of code loads in flight per lane (divides RB)
    static_assert(RB % D == 0, "ring depth must divide the batch");
    extern __shared__ __align__(16) unsigned char smem[];
    float4* xs = reinterpret_cast<float4*>(smem);                                   // [MT][nchunk][8] rotated
    float* xsum = reinterpret_cast<float*>(smem + (size_t)MT * a.nchunk * 8 * 16);  // [MT][nchunk]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t nbatch = (a.N + RB - 1) / RB;
    const int64_t bstride = (int64_t)gridDim.x * kW4Warps;
    const int64_t b0 = (int64_t)blockIdx.x * kW4Warps + warp;
    const int64_t nb_mine = b0 < nbatch ? (nbatch - 1 - b0) / bstride + 1 : 0;
    const int64_t T = nb_mine * RB;  // rows of this warp (the last batch may run past N)

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    auto row_of = [&](int64_t t) -> int64_t {
        const int64_t n = (b0 + (t / RB) * bstride) * RB + (t % RB);
        return n < a.N ? n : a.N - 1;
    };
    uint4 cw[D][CPL];
    uint32_t sb[D][CPL];  // scale | bias << 16 of the chunk's group
    auto issue = [&](int64_t t, int slot) {
        const int64_t n = row_of(t);
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const int c = lane + 32 * j;
            if (c < a.nchunk) {
                cw[slot][j] = __ldg(a.codes + n * a.nchunk + c);
                const int g = (32 * c) / a.G;
                sb[slot][j] = (uint32_t)__ldg(a.scales + n * a.ng + g) | ((uint32_t)__ldg(a.biases + n * a.ng + g) << 16);
            }
        }
    };
#pragma unroll
    for (int u = 0; u < D; ++u)
        if (u < T) issue(u, u);

    // activations: written by the preceding kernel
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = threadIdx.x; i < MT * a.nchunk * 8; i += kW4Threads) {
        const int m = i / (a.nchunk * 8), r = i - m * a.nchunk * 8, c = r >> 3, p = r & 7;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m < a.M) {
            const uint2 h = __ldcg(reinterpret_cast<const uint2*>(a.X + (int64_t)(a.m0 + m) * a.K + 32 * c + 4 * p));
            v = make_float4(bf16f(h.x & 0xFFFFu), bf16f(h.x >> 16), bf16f(h.y & 0xFFFFu), bf16f(h.y >> 16));
        }
        xs[(m * a.nchunk + c) * 8 + ((p + c) & 7)] = v;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < MT * a.nchunk; i += kW4Threads) {
        const int c = i % a.nchunk;
        float s = 0.f;
        for (int p = 0; p < 8; ++p) {
            const float4 v = xs[i * 8 + ((p + c) & 7)];
            s += (v.x + v.y) + (v.z + v.w);
        }
        xsum[i] = s;
    }
    __syncthreads();

    const uint64_t neg_magic = f2_pack(-8388608.f, -8388608.f);
    for (int64_t tb = 0; tb < T; tb += RB) {
        float part[MT][RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int64_t t = tb + r;
            const int slot = r % D;
            uint4 w[CPL];
            uint32_t sbv[CPL];
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                w[j] = cw[slot][j];
                sbv[j] = sb[slot][j];
            }
            if (t + D < T) issue(t + D, slot);
#pragma unroll
            for (int m = 0; m < MT; ++m) part[m][r] = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                const int c = lane + 32 * j;
                if (c < a.nchunk) {
                    uint64_t acc[MT];
#pragma unroll
                    for (int m = 0; m < MT; ++m) acc[m] = 0ull;
                    const uint32_t wd[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t E = wd[i] & 0x0F0F0F0Fu;         // codes 8i, 8i+2, 8i+4, 8i+6
                        const uint32_t O = (wd[i] >> 4) & 0x0F0F0F0Fu;  // codes 8i+1, 8i+3, 8i+5, 8i+7
#pragma unroll
                        for (int h = 0; h < 2; ++h) {  // piece 2i + h: columns 8i + 4h .. 8i + 4h + 3
                            const int p = 2 * i + h;
                            const uint64_t q01 = f2_add(f2_pack(__uint_as_float(prmt32(E, 0x4B000000u, 0x7650u | (2 * h))),
                                                                __uint_as_float(prmt32(O, 0x4B000000u, 0x7650u | (2 * h)))),
                                                        neg_magic);
                            const uint64_t q23 = f2_add(f2_pack(__uint_as_float(prmt32(E, 0x4B000000u, 0x7651u + 2 * h)),
                                                                __uint_as_float(prmt32(O, 0x4B000000u, 0x7651u + 2 * h))),
                                                        neg_magic);
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                const float4 x = xs[(m * a.nchunk + c) * 8 + ((p + c) & 7)];
                                acc[m] = f2_fma(q01, f2_pack(x.x, x.y), acc[m]);
                                acc[m] = f2_fma(q23, f2_pack(x.z, x.w), acc[m]);
                            }
                        }
                    }
                    const float s = bf16f(sbv[j] & 0xFFFFu), b = bf16f(sbv[j] >> 16);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float2 v = f2_unpack(acc[m]);
                        part[m][r] = fmaf(s, v.x + v.y, fmaf(b, xsum[m * a.nchunk + c], part[m][r]));
                    }
                }
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float tot = w4_reduce<RB>(part[m], lane);
            if (lane < RB && m < a.M) {
                const int64_t n = (b0 + (tb / RB) * bstride) * RB + lane;
                if (n < a.N) {
                    const int64_t o = (int64_t)(a.m0 + m) * a.N + n;
                    if (a.y_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[o] = __float2bfloat16_rn(tot);
                    else reinterpret_cast<float*>(a.Y)[o] = tot;
                }
            }
        }
    }
}

// Any G with G % 8 == 0 and K % G == 0: one warp per row, lanes over 32-bit
// words, each group's dot product and X sum formed in fp32.
__global__ void __launch_bounds__(256) gemv_w4_rows_kernel(const uint16_t* __restrict__ X, int M,
                                                          const uint32_t* __restrict__ codes,
                                                          const uint16_t* __restrict__ scales,
                                                          const uint16_t* __restrict__ biases, int64_t N, int K,
                                                          int G, void* Y, int y_bf16) {
    const int lane = threadIdx.x & 31;
    const int ng = K / G, words = K / 8;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int64_t wr = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; wr < N * M;
         wr += ((int64_t)gridDim.x * blockDim.x) / 32) {
        const int64_t n = wr % N;
        const int m = (int)(wr / N);
        const uint16_t* x = X + (int64_t)m * K;
        float y = 0.f;
        for (int g = 0; g < ng; ++g) {
            float dq = 0.f, dx = 0.f;
            for (int wi = lane; wi < G / 8; wi += 32) {
                const uint32_t word = __ldg(codes + n * words + (int64_t)g * (G / 8) + wi);
                for (int k = 0; k < 8; ++k) {
                    const float xv = bf16f(__ldg(x + (int64_t)g * G + 8 * wi + k));
                    dq = fmaf((float)((word >> (4 * k)) & 0xFu), xv, dq);
                    dx += xv;
                }
            }
            for (int o = 16; o >= 1; o >>= 1) {
                dq += __shfl_xor_sync(0xffffffffu, dq, o);
                dx += __shfl_xor_sync(0xffffffffu, dx, o);
            }
            y = fmaf(bf16f(__ldg(scales + n * ng + g)), dq, fmaf(bf16f(__ldg(biases + n * ng + g)), dx, y));
        }
        if (lane == 0) {
            const int64_t o = (int64_t)m * N + n;
            if (y_bf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(y);
            else reinterpret_cast<float*>(Y)[o] = y;
        }
    }
}

template <int MT, int CPL>
cudaError_t launch_w4(const W4Args& a, cudaStream_t stream, int sm_count) {
    auto kern = gemv_w4_kernel<MT, CPL>;
    const size_t smem = (size_t)MT * a.nchunk * (8 * 16 + 4);
    static SmemAttr smem_attr;
    if (smem > 48 * 1024)
        if (cudaError_t e = smem_attr.ensure(kern, (int)smem)) return e;
    constexpr int RB = w4_rb<MT>();
    const int64_t nbatch = (a.N + RB - 1) / RB;
    int64_t grid = (nbatch + kW4Warps - 1) / kW4Warps;
    if (grid > (MT <= 2 ? 2 : 1) * sm_count) grid = (MT <= 2 ? 2 : 1) * sm_count;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kW4Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int CPL>
cudaError_t launch_w4_mt(const W4Args& a, cudaStream_t stream, int sm_count) {
    switch (a.M) {
        case 1: return launch_w4<1, CPL>(a, stream, sm_count);
        case 2: return launch_w4<2, CPL>(a, stream, sm_count);
        case 3:
        case 4: return launch_w4<4, CPL>(a, stream, sm_count);
        default: return launch_w4<8, CPL>(a, stream, sm_count);
    }
}

}  // namespace

// Y = X . W^T for the W4A16 format, any M >= 1 (eight tokens per launch).
cudaError_t launch_gemv_w4(const uint16_t* X, int64_t M, const uint32_t* codes, const uint16_t* scales,
                           const uint16_t* biases, int64_t N, int64_t K, int G, void* Y, int y_bf16,
                           cudaStream_t stream, int sm_count) {
    const bool fast = G % 32 == 0 && K % 32 == 0 && K <= 4096 && (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
    if (!fast) {
        if (K > (1 << 30)) return cudaErrorNotSupported;
        int64_t grid = (N * M * 32 + 255) / 256;
        if (grid > 16 * sm_count) grid = 16 * sm_count;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, gemv_w4_rows_kernel, X, (int)M, codes, scales, biases, N, (int)K, G, Y, y_bf16);
    }
    W4Args a{};
    a.codes = reinterpret_cast<const uint4*>(codes);
    a.scales = scales;
    a.biases = biases;
    a.N = N;
    a.K = (int)K;
    a.G = G;
    a.ng = (int)(K / G);
    a.nchunk = (int)(K / 32);
    a.Y = Y;
    a.y_bf16 = y_bf16;
    const int cpl = (a.nchunk + 31) / 32;
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        a.X = X;
        a.m0 = (int)m0;
        a.M = (int)(M - m0 < 8 ? M - m0 : 8);
        cudaError_t e = cpl == 1   ? launch_w4_mt<1>(a, stream, sm_count)
                        : cpl == 2 ? launch_w4_mt<2>(a, stream, sm_count)
                                   : launch_w4_mt<4>(a, stream, sm_count);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace tq
