// gemv.cu -- fused unpack-and-scale matmul on the CUDA cores (decode path).
//
// tiny-llm "Week 2 Day 3: Quantize the Model", "Mathematical Formulation" and
// "Computation Flow": Y[m][n] = sum_g scale[n][g] * sum_{j in g} q[n][j] X[m][j]
// (bias 0, q = trit), the scale applied once per group ("SIMD Matvec" stage),
// accumulated in fp32.  The decoded scale is RNE_bf16(binary16 scale), the
// same magnitude the bf16 decoder writes.
//
// Row kernel: one warp per output row n; lane l walks the row's code bytes
// l, l+32, ...; each byte contributes its five trits against the activations
// staged in shared memory as bf16.  A row whose codes or scales fail
// validation produces NaN.
#include <atomic>

#include "tq_internal.cuh"

namespace tq {

constexpr int kGemvWarps = 8;
constexpr int kGemvMaxMT = 8;  // activation rows per pass

template <int MT>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_row_kernel(
    const uint16_t* __restrict__ X, int M, const uint8_t* __restrict__ codes,
    const uint16_t* __restrict__ scales, int64_t N, int K, int G, void* __restrict__ Y,
    int y_bf16, uint32_t* __restrict__ d_err) {
    extern __shared__ __align__(16) uint16_t xs[];  // [MT][K + 8] bf16, zero tail
    const int KP = K + 8;
    const int B = bytes_per_group(G);
    const int ng = K / G;
    const int row_bytes = ng * B;
    const int real = G - 5 * (B - 1);
    const uint32_t pmask = padding_mask(real), pones = padding_ones(real);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t err_acc = 0;

    for (int m0 = 0; m0 < M; m0 += MT) {
        const int mt = min(MT, M - m0);
        __syncthreads();
        for (int i = threadIdx.x; i < MT * KP; i += blockDim.x) {
            const int r = i / KP, k = i - r * KP;
            xs[i] = (r < mt && k < K) ? X[(int64_t)(m0 + r) * K + k] : (uint16_t)0;
        }
        __syncthreads();
        for (int64_t n = (int64_t)blockIdx.x * kGemvWarps + warp; n < N;
             n += (int64_t)gridDim.x * kGemvWarps) {
            const uint8_t* crow = codes + n * row_bytes;
            const uint16_t* srow = scales + n * ng;
            float acc[MT];
#pragma unroll
            for (int r = 0; r < MT; ++r) acc[r] = 0.f;
            uint32_t bad = 0;
            for (int c = lane; c < row_bytes; c += 32) {
                const int g = c / B, q = c - g * B;
                const uint32_t s = __ldg(srow + g);
                if (scale_is_bad(s)) bad |= TQ_DERR_SCALE;
                const float sc = __uint_as_float(scale_to_bf16_bits((uint16_t)s) << 16);
                uint32_t b = __ldg(crow + c);
                if (b >= 243) { bad |= TQ_DERR_BYTE; continue; }
                uint32_t digits = 0;
#pragma unroll
                for (int i = 0; i < 5; ++i) { digits |= (b % 3) << (2 * i); b /= 3; }
                if (q == B - 1 && (digits & pmask) != pones) bad |= TQ_DERR_PADDING;
                const int x0 = g * G + 5 * q;
#pragma unroll
                for (int r = 0; r < MT; ++r) {
                    const uint16_t* xr = xs + r * KP + x0;
                    float p = 0.f;
#pragma unroll
                    for (int i = 0; i < 5; ++i) {
                        const uint32_t d = (digits >> (2 * i)) & 3u;
                        const float xv = __uint_as_float((uint32_t)xr[i] << 16);
                        p += (d == 2u) ? xv : ((d == 0u) ? -xv : 0.f);
                    }
                    acc[r] = fmaf(sc, p, acc[r]);
                }
            }
            bad = __reduce_or_sync(0xffffffffu, bad);
#pragma unroll
            for (int r = 0; r < MT; ++r) {
                float v = acc[r];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                acc[r] = bad ? __uint_as_float(0x7FC00000u) : v;
            }
            if (lane == 0) {
                for (int r = 0; r < mt; ++r) {
                    const int64_t o = (int64_t)(m0 + r) * N + n;
                    if (y_bf16) reinterpret_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(acc[r]);
                    else reinterpret_cast<float*>(Y)[o] = acc[r];
                }
                err_acc |= bad;
            }
        }
    }
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

// Raises a kernel's dynamic shared memory limit only when a launch needs more
// than any earlier one, so steady-state launches (and stream capture) make no
// attribute calls.  The slot is per process; all devices here are B200s.
static std::atomic<int> smem_attr_slot[kGemvMaxMT + 1];

static cudaError_t ensure_smem_attr(const void* fn, std::atomic<int>& slot, size_t smem) {
    if ((int)smem <= 48 * 1024 || (int)smem <= slot.load(std::memory_order_acquire)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) {
        int cur = slot.load();
        while ((int)smem > cur && !slot.compare_exchange_weak(cur, (int)smem)) {
        }
    }
    return e;
}

size_t gemv_row_smem_bytes(int mt, int64_t K) { return (size_t)mt * (size_t)(K + 8) * 2; }

cudaError_t launch_gemv_rows(const uint16_t* X, int64_t M, const uint8_t* codes,
                             const uint16_t* scales, int64_t N, int64_t K, int G, void* Y,
                             int y_bf16, uint32_t* d_err, cudaStream_t stream, int sm_count,
                             size_t smem_limit) {
    int mt = (int)(M < kGemvMaxMT ? M : kGemvMaxMT);
    while (mt > 1 && gemv_row_smem_bytes(mt, K) > smem_limit) --mt;
    if (gemv_row_smem_bytes(mt, K) > smem_limit) return cudaErrorInvalidValue;
    const size_t smem = gemv_row_smem_bytes(mt, K);
    int64_t blocks = (N + kGemvWarps - 1) / kGemvWarps;
    const int64_t cap = (int64_t)sm_count * 8;
    if (blocks > cap) blocks = cap;
    const dim3 grid((unsigned)blocks), block(kGemvWarps * 32);
#define TQ_GEMV_CASE(T)                                                                         \
    case T: {                                                                                   \
        auto k = gemv_row_kernel<T>;                                                            \
        cudaError_t e = ensure_smem_attr((const void*)k, smem_attr_slot[T], smem);              \
        if (e != cudaSuccess) return e;                                                         \
        k<<<grid, block, smem, stream>>>(X, (int)M, codes, scales, N, (int)K, G, Y, y_bf16,     \
                                         d_err);                                                \
        return cudaGetLastError();                                                              \
    }
    switch (mt) {
        TQ_GEMV_CASE(1)
        TQ_GEMV_CASE(2)
        TQ_GEMV_CASE(3)
        TQ_GEMV_CASE(4)
        TQ_GEMV_CASE(5)
        TQ_GEMV_CASE(6)
        TQ_GEMV_CASE(7)
        TQ_GEMV_CASE(8)
        default:
            return cudaErrorInvalidValue;
    }
#undef TQ_GEMV_CASE
}

}  // namespace tq
