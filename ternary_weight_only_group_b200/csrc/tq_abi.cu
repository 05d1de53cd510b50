// tq_abi.cu -- extern "C" entry points of libtq: argument validation and
// kernel dispatch.  Every check here runs on the host before any launch; a
// failed check returns a status and enqueues nothing.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "tq_internal.cuh"

namespace tq {
cudaError_t launch_quantize_pack(const uint16_t* W, int64_t N, int64_t K, int G, uint8_t* codes,
                                 uint16_t* scales, uint32_t* d_err, cudaStream_t stream,
                                 int sm_count);
cudaError_t launch_unpack(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t K, int G,
                          uint16_t* out, uint32_t* d_err, cudaStream_t stream, int sm_count);
cudaError_t launch_gemv_rows(const uint16_t* X, int64_t M, const uint8_t* codes,
                             const uint16_t* scales, int64_t N, int64_t K, int G, void* Y,
                             int y_bf16, uint32_t* d_err, cudaStream_t stream, int sm_count,
                             size_t smem_limit);
cudaError_t launch_gemv_lut(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                            int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                            cudaStream_t stream, int sm_count, size_t smem_limit);
cudaError_t launch_gemv_lut_stream(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                                   int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                                   cudaStream_t stream, int sm_count, int fmt);
cudaError_t launch_gemv_w4(const uint16_t* X, int64_t M, const uint32_t* codes, const uint16_t* scales,
                           const uint16_t* biases, int64_t N, int64_t K, int G, void* Y, int y_bf16,
                           cudaStream_t stream, int sm_count);
cudaError_t launch_gemv_lut_stream_w4(const uint16_t* X, int64_t M, const uint32_t* codes, const uint16_t* scales,
                                      const uint16_t* biases, int64_t N, int64_t K, int G, void* Y, int y_bf16,
                                      cudaStream_t stream, int sm_count);
cudaError_t launch_gemv_predecode(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                                  int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                                  cudaStream_t stream, int sm_count, int fmt);
cudaError_t launch_gemm_small(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                              int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                              cudaStream_t stream, int sm_count, bool* handled, int fmt, const uint16_t* biases = nullptr);
cudaError_t launch_quantize_pack2(const uint16_t* W, int64_t N, int64_t K, int G, uint8_t* codes,
                                  uint16_t* scales, uint32_t* d_err, cudaStream_t stream, int sm_count);
cudaError_t launch_unpack2(const uint8_t* codes, const uint16_t* scales, int64_t N, int64_t K, int G, uint16_t* out,
                           uint32_t* d_err, cudaStream_t stream, int sm_count);
cudaError_t launch_gemv2(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales, int64_t N,
                         int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err, cudaStream_t stream, int sm_count);
cudaError_t launch_gemm_tc(const uint16_t* X, int64_t M, const uint8_t* codes,
                           const uint16_t* scales, int64_t N, int64_t K, int G, void* Y,
                           int y_bf16, uint32_t* d_err, cudaStream_t stream, int sm_count,
                           bool* handled, int fmt, const uint16_t* biases = nullptr);

namespace {

struct DeviceInfo {
    int sm_count = 0;
    int major = 0, minor = 0;
    size_t smem_optin = 0;
    bool ok = false;
};

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
DeviceInfo g_dev[kMaxDevices];

tq_status device_info(const DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return TQ_ERR_CUDA;
    }
    std::call_once(g_dev_once[dev], [dev] {
        DeviceInfo& d = g_dev[dev];
        int smem = 0;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess) {
            d.smem_optin = (size_t)smem;
            d.ok = true;
        } else {
            cudaGetLastError();
        }
    });
    const DeviceInfo& d = g_dev[dev];
    if (!d.ok) return TQ_ERR_CUDA;
    // The kernels are built for sm_100a only.
    if (d.major != 10 || d.minor != 0) return TQ_ERR_UNSUPPORTED;
    *out = &d;
    return TQ_OK;
}

bool shape_ok(int64_t N, int64_t K, int G) {
    if (G < 1 || G > TQ_MAX_G) return false;
    if (N < 0 || K < 0 || K % G != 0) return false;
    if (N > 0 && K > (int64_t(1) << 62) / N) return false;
    return true;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    if (!na || !nb) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

tq_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return TQ_OK;
    cudaGetLastError();
    return TQ_ERR_CUDA;
}

struct MatmulArgs {
    const void* X;
    int64_t M;
    const uint8_t* codes;
    const void* scales;
    int64_t N, K;
    int G;
    void* Y;
    tq_out_dtype yt;
    int fmt = 3;  // 3: base-3 codes, 2: 2-bit codes
};

tq_status check_matmul(const MatmulArgs& a) {
    if (!shape_ok(a.N, a.K, a.G) || a.M < 0) return TQ_ERR_INVALID_ARG;
    if (a.yt != TQ_OUT_F32 && a.yt != TQ_OUT_BF16) return TQ_ERR_INVALID_ARG;
    if (a.M > 0 && a.K > (int64_t(1) << 62) / a.M) return TQ_ERR_INVALID_ARG;
    if (a.M > 0 && a.N > (int64_t(1) << 62) / a.M) return TQ_ERR_INVALID_ARG;
    const size_t cb = a.fmt == 2 ? tq2_codes_bytes(a.N, a.K, a.G) : tq_codes_bytes(a.N, a.K, a.G);
    const size_t sb = tq_scales_bytes(a.N, a.K, a.G);
    const size_t xb = (size_t)a.M * (size_t)a.K * 2;
    const size_t yb = (size_t)a.M * (size_t)a.N * (a.yt == TQ_OUT_F32 ? 4 : 2);
    if ((xb && !a.X) || (cb && !a.codes) || (sb && !a.scales) || (yb && !a.Y)) return TQ_ERR_INVALID_ARG;
    if (overlap(a.Y, yb, a.X, xb) || overlap(a.Y, yb, a.codes, cb) || overlap(a.Y, yb, a.scales, sb))
        return TQ_ERR_INVALID_ARG;
    if (!aligned(a.X, 16) || !aligned(a.scales, 2) || !aligned(a.Y, a.yt == TQ_OUT_F32 ? 4 : 2))
        return TQ_ERR_ALIGNMENT;
    if (a.fmt == 2 && !aligned(a.codes, 4)) return TQ_ERR_ALIGNMENT;
    return TQ_OK;
}

// Y for K == 0: every output is an empty sum, +0.
tq_status zero_output(const MatmulArgs& a, cudaStream_t stream) {
    const size_t yb = (size_t)a.M * (size_t)a.N * (a.yt == TQ_OUT_F32 ? 4 : 2);
    return from_cuda(cudaMemsetAsync(a.Y, 0, yb, stream));
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" {

size_t tq_codes_bytes(int64_t N, int64_t K, int G) {
    if (!shape_ok(N, K, G)) return 0;
    return (size_t)N * (size_t)(K / G) * (size_t)bytes_per_group(G);
}

size_t tq_scales_bytes(int64_t N, int64_t K, int G) {
    if (!shape_ok(N, K, G)) return 0;
    return (size_t)N * (size_t)(K / G) * 2;
}

size_t tq_workspace_bytes(int64_t M, int64_t N, int64_t K, int G) {
    (void)M; (void)N; (void)K; (void)G;
    return 0;
}

tq_status tq_quantize_pack(const void* W, int64_t N, int64_t K, int G, uint8_t* codes, void* scales,
                           uint32_t* d_err, tq_stream_t stream) {
    if (!shape_ok(N, K, G)) return TQ_ERR_INVALID_ARG;
    const size_t wb = (size_t)N * (size_t)K * 2;
    const size_t cb = tq_codes_bytes(N, K, G), sb = tq_scales_bytes(N, K, G);
    if ((wb && !W) || (cb && !codes) || (sb && !scales)) return TQ_ERR_INVALID_ARG;
    if (overlap(codes, cb, W, wb) || overlap(scales, sb, W, wb) || overlap(codes, cb, scales, sb))
        return TQ_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(scales, 2)) return TQ_ERR_ALIGNMENT;
    if (wb == 0) return TQ_OK;
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    return from_cuda(launch_quantize_pack(static_cast<const uint16_t*>(W), N, K, G, codes,
                                          static_cast<uint16_t*>(scales), d_err,
                                          (cudaStream_t)stream, d->sm_count));
}

tq_status tq_unpack_bf16(const uint8_t* codes, const void* scales, int64_t N, int64_t K, int G,
                         void* W_out, uint32_t* d_err, tq_stream_t stream) {
    if (!shape_ok(N, K, G)) return TQ_ERR_INVALID_ARG;
    const size_t wb = (size_t)N * (size_t)K * 2;
    const size_t cb = tq_codes_bytes(N, K, G), sb = tq_scales_bytes(N, K, G);
    if ((wb && !W_out) || (cb && !codes) || (sb && !scales)) return TQ_ERR_INVALID_ARG;
    if (overlap(W_out, wb, codes, cb) || overlap(W_out, wb, scales, sb)) return TQ_ERR_INVALID_ARG;
    if (!aligned(W_out, 16) || !aligned(scales, 2)) return TQ_ERR_ALIGNMENT;
    if (wb == 0) return TQ_OK;
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    return from_cuda(launch_unpack(codes, static_cast<const uint16_t*>(scales), N, K, G,
                                   static_cast<uint16_t*>(W_out), d_err, (cudaStream_t)stream,
                                   d->sm_count));
}

// The streaming one-token kernel once per token row (X row m -> Y row m), for
// M <= kStreamMaxTokens.  One token always; 2..4 tokens only from
// kStreamMinWeightsMulti weights, where M passes over the weights still beat
// the multi-token kernels (172032 x 1024: 14.3 us per pass).  Returns
// cudaErrorNotSupported, having launched nothing, when the kernel does not
// cover the shape.
constexpr int64_t kStreamMaxTokens = 4;
// tq_w4_gemv: whether the streaming lookup-table kernel, once per token,
// beats the CUDA-core kernel (all tokens in one pass).  Measured on B200:
// one token from about 12 Mi weights (6 Mi at K >= 2048): 14336 x 1024 5.8
// us against 6.1, 8192 x 1024 5.5 against 4.3, 4096 x 2048 5.7 against 9.2;
// 2..4 tokens where the CUDA-core kernel has few 32-column chunks per row
// (K <= 512: 65536 x 512 at 4 tokens 32 us against 50) or from 96 Mi weights
// (172032 x 1024 at 4 tokens 112 us against 132; 57344 x 1024 49 against 48).
constexpr int64_t kW4StreamMaxTokens = 4;
static bool w4_stream_wins(int64_t M, int64_t N, int64_t K) {
    const int64_t nk = N * K;
    if (M < 1 || M > kW4StreamMaxTokens || nk < (K >= 2048 ? (int64_t)6 << 20 : (int64_t)12 << 20)) return false;
    return M == 1 || K <= 512 || nk >= (int64_t)96 << 20;
}
constexpr int64_t kStreamMinWeightsMulti = (int64_t)48 << 20;
static cudaError_t stream_per_token(const void* X, int64_t M, const uint8_t* codes, const void* scales, int64_t N,
                                    int64_t K, int G, void* Y, tq_out_dtype yt, uint32_t* d_err, cudaStream_t stream,
                                    int sm_count, int fmt) {
    if (M > kStreamMaxTokens || (M > 1 && N * K < kStreamMinWeightsMulti)) return cudaErrorNotSupported;
    const size_t ysz = yt == TQ_OUT_BF16 ? 2 : 4;
    for (int64_t m = 0; m < M; ++m) {
        const cudaError_t e = launch_gemv_lut_stream(static_cast<const uint16_t*>(X) + m * K, 1, codes,
                                                     static_cast<const uint16_t*>(scales), N, K, G,
                                                     static_cast<char*>(Y) + (size_t)m * N * ysz, yt == TQ_OUT_BF16,
                                                     d_err, stream, sm_count, fmt);
        if (e != cudaSuccess) return e;  // NotSupported can only come from the first (same shape every time)
    }
    return cudaSuccess;
}

tq_status tq_gemv(const void* X, int64_t M, const uint8_t* codes, const void* scales, int64_t N,
                  int64_t K, int G, void* Y, tq_out_dtype yt, void* workspace, size_t ws_bytes,
                  uint32_t* d_err, tq_stream_t stream) {
    (void)workspace; (void)ws_bytes;
    const MatmulArgs a{X, M, codes, scales, N, K, G, Y, yt};
    if (tq_status st = check_matmul(a)) return st;
    if (M == 0 || N == 0) return TQ_OK;
    if (K == 0) return zero_output(a, (cudaStream_t)stream);  // empty sums
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    // 1..4 tokens (1..8 where the tensor path below does not take the
    // shape), matrix small enough for one or two CTAs per SM to hold its
    // decoded rows: weights decoded before the activations are awaited.  At
    // 5..8 tokens the tensor path is faster (M-sweep, 28 layers of 1536-4096
    // wide projections at 8 tokens: 5.7 us per launch against 6.9)
    cudaError_t e = cudaErrorNotSupported;
    if (M <= 4 || G % 64 != 0 || K % 64 != 0) {
        e = launch_gemv_predecode(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales),
                                  N, K, G, Y, yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count, 3);
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
    }
    // 1..4 tokens over a larger matrix: lookup tables of one 512-column K
    // slice per CTA, slices spread over a cluster, code words streamed per
    // lane; one launch per token (172032 x 1024: 14.3 us per token, against
    // 49 us for two tokens on the lookup-table kernel below and 88 us for the
    // tensor-core path at 3..16 tokens)
    if (M <= kStreamMaxTokens) {
        e = stream_per_token(X, M, codes, scales, N, K, G, Y, yt, d_err, (cudaStream_t)stream, d->sm_count, 3);
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
    }
    auto lut = [&]() {
        return launch_gemv_lut(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales), N,
                               K, G, Y, yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count, d->smem_optin);
    };
    // 1..2 tokens: lookup tables (faster than the tensor path at these M on
    // large matrices: 172032 x 1024, M=2: 49 us against 100 us)
    if (M <= 2) {
        e = lut();
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
    }
    // 3..64 tokens: the tensor-core small-M kernels (M=4 on 172032 x 1024:
    // 100 us against 455 us with lookup tables)
    {
        bool handled = false;
        e = launch_gemm_small(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales), N,
                              K, G, Y, yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count, &handled, 3);
        if (e != cudaSuccess) return from_cuda(e);
        if (handled) return TQ_OK;
    }
    if (M > 2) {  // shapes the tensor path does not cover
        e = lut();
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
    }
    e = launch_gemv_rows(static_cast<const uint16_t*>(X), M, codes,
                         static_cast<const uint16_t*>(scales), N, K, G, Y,
                         yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count,
                         d->smem_optin);
    if (e == cudaErrorInvalidValue) return TQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

tq_status tq_gemm(const void* X, int64_t M, const uint8_t* codes, const void* scales, int64_t N,
                  int64_t K, int G, void* Y, tq_out_dtype yt, void* workspace, size_t ws_bytes,
                  uint32_t* d_err, tq_stream_t stream) {
    (void)workspace; (void)ws_bytes;
    const MatmulArgs a{X, M, codes, scales, N, K, G, Y, yt};
    if (tq_status st = check_matmul(a)) return st;
    if (M == 0 || N == 0) return TQ_OK;
    if (K == 0) return zero_output(a, (cudaStream_t)stream);  // empty sums
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    bool handled = false;
    cudaError_t e = cudaSuccess;
    if (M <= 64)
        e = launch_gemm_small(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales), N,
                              K, G, Y, yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count, &handled, 3);
    if (e == cudaSuccess && !handled)
        e = launch_gemm_tc(static_cast<const uint16_t*>(X), M, codes,
                           static_cast<const uint16_t*>(scales), N, K, G, Y,
                           yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count,
                           &handled, 3);
    if (e != cudaSuccess) return from_cuda(e);
    if (!handled) return TQ_ERR_UNSUPPORTED;
    return TQ_OK;
}

// ---- 2-bit ternary format

size_t tq2_codes_bytes(int64_t N, int64_t K, int G) {
    if (!shape_ok(N, K, G)) return 0;
    return (size_t)N * (size_t)(K / G) * (size_t)((G + 3) / 4);
}

tq_status tq2_quantize_pack(const void* W, int64_t N, int64_t K, int G, uint8_t* codes, void* scales,
                            uint32_t* d_err, tq_stream_t stream) {
    if (!shape_ok(N, K, G)) return TQ_ERR_INVALID_ARG;
    const size_t wb = (size_t)N * (size_t)K * 2;
    const size_t cb = tq2_codes_bytes(N, K, G), sb = tq_scales_bytes(N, K, G);
    if ((wb && !W) || (cb && !codes) || (sb && !scales)) return TQ_ERR_INVALID_ARG;
    if (overlap(codes, cb, W, wb) || overlap(scales, sb, W, wb) || overlap(codes, cb, scales, sb))
        return TQ_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(scales, 2) || !aligned(codes, 4)) return TQ_ERR_ALIGNMENT;
    if (wb == 0) return TQ_OK;
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    return from_cuda(launch_quantize_pack2(static_cast<const uint16_t*>(W), N, K, G, codes,
                                           static_cast<uint16_t*>(scales), d_err, (cudaStream_t)stream,
                                           d->sm_count));
}

tq_status tq2_unpack_bf16(const uint8_t* codes, const void* scales, int64_t N, int64_t K, int G, void* W_out,
                          uint32_t* d_err, tq_stream_t stream) {
    if (!shape_ok(N, K, G)) return TQ_ERR_INVALID_ARG;
    const size_t wb = (size_t)N * (size_t)K * 2;
    const size_t cb = tq2_codes_bytes(N, K, G), sb = tq_scales_bytes(N, K, G);
    if ((wb && !W_out) || (cb && !codes) || (sb && !scales)) return TQ_ERR_INVALID_ARG;
    if (overlap(W_out, wb, codes, cb) || overlap(W_out, wb, scales, sb)) return TQ_ERR_INVALID_ARG;
    if (!aligned(W_out, 16) || !aligned(scales, 2) || !aligned(codes, 4)) return TQ_ERR_ALIGNMENT;
    if (wb == 0) return TQ_OK;
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    return from_cuda(launch_unpack2(codes, static_cast<const uint16_t*>(scales), N, K, G,
                                    static_cast<uint16_t*>(W_out), d_err, (cudaStream_t)stream, d->sm_count));
}

tq_status tq2_gemv(const void* X, int64_t M, const uint8_t* codes, const void* scales, int64_t N, int64_t K, int G,
                   void* Y, tq_out_dtype yt, void* workspace, size_t ws_bytes, uint32_t* d_err,
                   tq_stream_t stream) {
    (void)workspace; (void)ws_bytes;
    MatmulArgs a{X, M, codes, scales, N, K, G, Y, yt};
    a.fmt = 2;
    if (tq_status st = check_matmul(a)) return st;
    if (M == 0 || N == 0) return TQ_OK;
    if (K == 0) return zero_output(a, (cudaStream_t)stream);  // empty sums
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    // 1..4 tokens over a large matrix: the streaming lookup-table kernel once
    // per token, as tq_gemv (its fixed cost, the table build after the
    // activations arrive, loses to the CUDA-core kernel below about 24 M
    // weights at K <= 1536 and 8 M weights above: 14336 x 1024 takes 6.0 us
    // against 7.7 us, 28672 x 1024 9.7 us against 7.9 us, 3584 x 3584 10.9
    // us against 7.8 us)
    const bool big = K >= 2048 ? N * K >= (int64_t)(8 << 20) : N * K >= (int64_t)(24 << 20);
    if (M <= kStreamMaxTokens && big) {
        const cudaError_t e = stream_per_token(X, M, codes, scales, N, K, G, Y, yt, d_err, (cudaStream_t)stream,
                                               d->sm_count, 2);
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
    }
    // 1..4 tokens (1..8 where the tensor path does not take the shape), matrix
    // small enough for one or two CTAs per SM to hold its decoded rows: the
    // pre-decode kernel, weights decoded before the activations are awaited
    // (the headline's FFN projections: 4.8 us per launch on the CUDA-core
    // kernel below in a chain of dependent launches)
    if (M <= 4 || G % 64 != 0 || K % 64 != 0) {
        const cudaError_t e = launch_gemv_predecode(static_cast<const uint16_t*>(X), M, codes,
                                                    static_cast<const uint16_t*>(scales), N, K, G, Y,
                                                    yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count, 2);
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
    }
    // 3..64 tokens: the tensor-core small-M kernels on the 2-bit codes
    if (M >= 3) {
        bool handled = false;
        const cudaError_t e = launch_gemm_small(static_cast<const uint16_t*>(X), M, codes,
                                                static_cast<const uint16_t*>(scales), N, K, G, Y, yt == TQ_OUT_BF16,
                                                d_err, (cudaStream_t)stream, d->sm_count, &handled, 2);
        if (e != cudaSuccess) return from_cuda(e);
        if (handled) return TQ_OK;
    }
    const cudaError_t e = launch_gemv2(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales),
                                       N, K, G, Y, yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count);
    if (e == cudaErrorNotSupported) return TQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

tq_status tq2_gemm(const void* X, int64_t M, const uint8_t* codes, const void* scales, int64_t N, int64_t K, int G,
                   void* Y, tq_out_dtype yt, void* workspace, size_t ws_bytes, uint32_t* d_err,
                   tq_stream_t stream) {
    (void)workspace; (void)ws_bytes;
    MatmulArgs a{X, M, codes, scales, N, K, G, Y, yt};
    a.fmt = 2;
    if (tq_status st = check_matmul(a)) return st;
    if (M == 0 || N == 0) return TQ_OK;
    if (K == 0) return zero_output(a, (cudaStream_t)stream);  // empty sums
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    bool handled = false;
    cudaError_t e = cudaSuccess;
    if (M <= 64)
        e = launch_gemm_small(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales), N, K, G,
                              Y, yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count, &handled, 2);
    if (e == cudaSuccess && !handled)
        e = launch_gemm_tc(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales), N, K, G, Y,
                           yt == TQ_OUT_BF16, d_err, (cudaStream_t)stream, d->sm_count, &handled, 2);
    if (e != cudaSuccess) return from_cuda(e);
    if (!handled) return TQ_ERR_UNSUPPORTED;
    return TQ_OK;
}

// ---- W4A16 affine format

size_t tq_w4_codes_bytes(int64_t N, int64_t K, int G) {
    if (!shape_ok(N, K, G) || G % 8 != 0) return 0;
    return (size_t)N * (size_t)(K / 8) * 4;
}

tq_status tq_w4_gemv(const void* X, int64_t M, const uint32_t* codes, const void* scales, const void* biases,
                     int64_t N, int64_t K, int G, void* Y, tq_out_dtype yt, tq_stream_t stream) {
    if (!shape_ok(N, K, G) || G % 8 != 0 || M < 0) return TQ_ERR_INVALID_ARG;
    if (yt != TQ_OUT_F32 && yt != TQ_OUT_BF16) return TQ_ERR_INVALID_ARG;
    if (M > 0 && (K > (int64_t(1) << 62) / M || N > (int64_t(1) << 62) / M)) return TQ_ERR_INVALID_ARG;
    const size_t cb = tq_w4_codes_bytes(N, K, G), sb = tq_scales_bytes(N, K, G);
    const size_t xb = (size_t)M * (size_t)K * 2;
    const size_t yb = (size_t)M * (size_t)N * (yt == TQ_OUT_F32 ? 4 : 2);
    if ((xb && !X) || (cb && !codes) || (sb && (!scales || !biases)) || (yb && !Y)) return TQ_ERR_INVALID_ARG;
    if (overlap(Y, yb, X, xb) || overlap(Y, yb, codes, cb) || overlap(Y, yb, scales, sb) || overlap(Y, yb, biases, sb))
        return TQ_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(codes, 4) || !aligned(scales, 2) || !aligned(biases, 2) ||
        !aligned(Y, yt == TQ_OUT_F32 ? 4 : 2))
        return TQ_ERR_ALIGNMENT;
    if (M == 0 || N == 0) return TQ_OK;
    if (K == 0) return from_cuda(cudaMemsetAsync(Y, 0, yb, (cudaStream_t)stream));  // empty sums
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    // 1..4 tokens over a large matrix: the streaming lookup-table kernel once
    // per token (tables of 256 columns per CTA)
    if (w4_stream_wins(M, N, K)) {
        const size_t ysz = yt == TQ_OUT_BF16 ? 2 : 4;
        cudaError_t e = cudaSuccess;
        for (int64_t m = 0; m < M && e == cudaSuccess; ++m)
            e = launch_gemv_lut_stream_w4(static_cast<const uint16_t*>(X) + m * K, 1, codes,
                                          static_cast<const uint16_t*>(scales), static_cast<const uint16_t*>(biases),
                                          N, K, G, static_cast<char*>(Y) + (size_t)m * N * ysz, yt == TQ_OUT_BF16,
                                          (cudaStream_t)stream, d->sm_count);
        if (e != cudaErrorNotSupported) return from_cuda(e);  // NotSupported only from the first launch
        cudaGetLastError();
    }
    // 5..64 tokens: the small-M tensor kernels (split-K for few row tiles,
    // persistent for many), each weight as two bf16 terms in tensor memory,
    // where they take the shape (M-sweep projections 1536 x 1536 .. 4096 x
    // 1536: 4.8-8.9 us at 16 tokens against 9.2-17.7 us for 8 tokens on the
    // CUDA-core kernel)
    if (M >= 5 && M <= 64) {
        bool handled = false;
        const cudaError_t e = launch_gemm_small(static_cast<const uint16_t*>(X), M,
                                                reinterpret_cast<const uint8_t*>(codes),
                                                static_cast<const uint16_t*>(scales), N, K, G, Y, yt == TQ_OUT_BF16,
                                                nullptr, (cudaStream_t)stream, d->sm_count, &handled, 4,
                                                static_cast<const uint16_t*>(biases));
        if (e != cudaSuccess) return from_cuda(e);
        if (handled) return TQ_OK;
    }
    const cudaError_t e = launch_gemv_w4(static_cast<const uint16_t*>(X), M, codes, static_cast<const uint16_t*>(scales),
                                         static_cast<const uint16_t*>(biases), N, K, G, Y, yt == TQ_OUT_BF16,
                                         (cudaStream_t)stream, d->sm_count);
    if (e == cudaErrorNotSupported) return TQ_ERR_UNSUPPORTED;
    return from_cuda(e);
}

tq_status tq_w4_gemm(const void* X, int64_t M, const uint32_t* codes, const void* scales, const void* biases,
                     int64_t N, int64_t K, int G, void* Y, tq_out_dtype yt, tq_stream_t stream) {
    if (!shape_ok(N, K, G) || G % 8 != 0 || M < 0) return TQ_ERR_INVALID_ARG;
    if (yt != TQ_OUT_F32 && yt != TQ_OUT_BF16) return TQ_ERR_INVALID_ARG;
    if (M > 0 && (K > (int64_t(1) << 62) / M || N > (int64_t(1) << 62) / M)) return TQ_ERR_INVALID_ARG;
    const size_t cb = tq_w4_codes_bytes(N, K, G), sb = tq_scales_bytes(N, K, G);
    const size_t xb = (size_t)M * (size_t)K * 2;
    const size_t yb = (size_t)M * (size_t)N * (yt == TQ_OUT_F32 ? 4 : 2);
    if ((xb && !X) || (cb && !codes) || (sb && (!scales || !biases)) || (yb && !Y)) return TQ_ERR_INVALID_ARG;
    if (overlap(Y, yb, X, xb) || overlap(Y, yb, codes, cb) || overlap(Y, yb, scales, sb) || overlap(Y, yb, biases, sb))
        return TQ_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(codes, 4) || !aligned(scales, 2) || !aligned(biases, 2) ||
        !aligned(Y, yt == TQ_OUT_F32 ? 4 : 2))
        return TQ_ERR_ALIGNMENT;
    if (M == 0 || N == 0) return TQ_OK;
    if (K == 0) return from_cuda(cudaMemsetAsync(Y, 0, yb, (cudaStream_t)stream));  // empty sums
    const DeviceInfo* d = nullptr;
    if (tq_status st = device_info(&d)) return st;
    bool handled = false;
    if (M <= 64) {  // small M: the small-M tensor kernels (W in tensor memory) where they take the shape
        const cudaError_t e = launch_gemm_small(static_cast<const uint16_t*>(X), M,
                                                reinterpret_cast<const uint8_t*>(codes),
                                                static_cast<const uint16_t*>(scales), N, K, G, Y, yt == TQ_OUT_BF16,
                                                nullptr, (cudaStream_t)stream, d->sm_count, &handled, 4,
                                                static_cast<const uint16_t*>(biases));
        if (e != cudaSuccess) return from_cuda(e);
        if (handled) return TQ_OK;
    }
    const cudaError_t e = launch_gemm_tc(static_cast<const uint16_t*>(X), M, reinterpret_cast<const uint8_t*>(codes),
                                         static_cast<const uint16_t*>(scales), N, K, G, Y, yt == TQ_OUT_BF16, nullptr,
                                         (cudaStream_t)stream, d->sm_count, &handled, 4,
                                         static_cast<const uint16_t*>(biases));
    if (e != cudaSuccess) return from_cuda(e);
    return handled ? TQ_OK : TQ_ERR_UNSUPPORTED;
}

const char* tq_status_string(tq_status s) {
    switch (s) {
        case TQ_OK: return "TQ_OK";
        case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
        case TQ_ERR_ALIGNMENT: return "TQ_ERR_ALIGNMENT";
        case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
        case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    }
    return "TQ_ERR_UNKNOWN";
}

const char* tq_version(void) { return "libtq 0.1 sm_100a"; }

}  // extern "C"
