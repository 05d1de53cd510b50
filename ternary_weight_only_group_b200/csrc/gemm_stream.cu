// gemm_stream.cu -- small-M fused matmul over many row tiles on the tensor
// cores (persistent, tcgen05, sm_100a).
//
// Same result as the decode GEMV (tiny-llm "Week 2 Day 3: Quantize the Model",
// "Mathematical Formulation": C = A B^T with B reconstructed per group, float
// accumulation), for 1 <= M <= 64 tokens and matrices with at least as many
// 128-row tiles as half the SMs, where splitting K over a cluster buys
// nothing.  One CTA per SM walks its tiles; each tile is
//   D^T[128 W rows x NT tokens] += What[128 x 16] . X[NT x 16]^T
// over K in 64-column stages, with What decoded on chip straight into tensor
// memory (a decoder thread owns one W row = one tensor-memory lane and
// stores a stage's 64 bf16 with tcgen05.st), where the MMA reads it as the A
// operand, and X stages loaded by TMA (NT = 16, 32 or 64 rows, zero-filled
// past M).
//   warp 0       TMA producer of the X stages
//   warp 1       MMA issuer (kind::f16, M=128, N=NT, fp32 accumulators in TMEM)
//   warp 2       tensor-memory allocation
//   warps 4-11   decoders: two groups of four warps on alternating stages,
//                one W row per thread; each thread fetches its own rows'
//                code windows and scales with cp.async three of its stages
//                ahead
//   warps 12-15  epilogue: two TMEM accumulators, so tile j is read out and
//                stored while tile j+1 accumulates; W rows whose first
//                token came out NaN are rescanned for the error bits
// All mbarrier waits are bounded (globaltimer deadline -> TQ_DERR_TIMEOUT).
#include <atomic>
#include <cstring>

#include "tc_common.cuh"

namespace tq {
namespace stream {

using namespace tc;

constexpr int WM = 128;  // W rows per tile (UMMA M)
constexpr int BK = 64;
constexpr int STAGES = 6;  // even: a stage slot always belongs to the same decoder group
constexpr int CR = 4;      // code windows in flight per decoder thread
constexpr int kThreads = 512;
constexpr int kDecWarp0 = 4, kEpiWarp0 = 12;
constexpr int kGroupWarps = 4;
constexpr uint32_t WIN = 48;  // per row: 32 code bytes, the 4-byte words holding the scale and (W4A16) the bias

// Tensor memory: two accumulators of NT columns, then one 32-column slot of
// decoded W (128 x 64 bf16) per stage.
template <int NT>
constexpr uint32_t kAccCols = 2 * NT;
// columns of a stage's W slot: 32 (64 bf16 of a row), 64 for W4A16 (hi and lo terms)
template <int FMT>
constexpr uint32_t kSlotCols = FMT == 4 ? 64 : 32;
template <int NT, int FMT>
constexpr uint32_t kTmemCols = kAccCols<NT> + kSlotCols<FMT> * STAGES <= 256 ? 256 : 512;

template <int NT>
struct Smem {
    uint8_t x[STAGES][NT * 128];    // X stages (UMMA B): NT rows of 128 bytes, 1024-byte aligned
    uint8_t win[2][CR][WM * WIN];   // code windows + scales, per decoder group
    uint32_t lut[256 * 32];           // byte -> PRMT selectors of its digits 0..3, one copy per lane
    uint64_t full_x[STAGES], full_w[STAGES], empty[STAGES];
    uint64_t tfull[2], tempty[2], done;
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    const uint8_t* codes;
    const uint8_t* codes_end;
    int64_t row_bytes;
    const uint16_t* scales;
    const uint16_t* scales_end;
    const uint16_t* biases;  // W4A16 only
    const uint16_t* biases_end;
    void* Y;
    uint32_t* d_err;
    int64_t M, N;
    int K, G, B, ng;
    int tiles;
    int y_bf16;
    uint32_t pad_base, pad_span;  // canonical range of a group's last code byte
    WaitCfg wc;                   // wait bound and the withheld-load test hook
};

__device__ __forceinline__ void cp_async16(uint8_t* dst, const uint8_t* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s32(dst)), "l"(__cvta_generic_to_global(src))
                 : "memory");
}
__device__ __forceinline__ void cp_async4(uint8_t* dst, const uint8_t* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s32(dst)), "l"(__cvta_generic_to_global(src))
                 : "memory");
}

// The 32 bytes from (A rounded down to 16) into dst; pieces that fall outside
// [begin, end) are not read (bytes inside it are copied one by one there).
__device__ __forceinline__ void fetch_window(uint8_t* dst, const uint8_t* A, const uint8_t* begin,
                                             const uint8_t* end) {
    const uint8_t* a = reinterpret_cast<const uint8_t*>(reinterpret_cast<uintptr_t>(A) & ~(uintptr_t)15);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const uint8_t* src = a + 16 * c;
        if (src >= begin && src + 16 <= end) {
            cp_async16(dst + 16 * c, src);
        } else {
            for (int b = 0; b < 16; ++b)
                if (src + b >= begin && src + b < end) dst[16 * c + b] = src[b];
        }
    }
}

// The aligned 4-byte word holding the scale at S (2-byte aligned) into dst,
// or the scale alone (at dst + (S & 2)) when that word leaves [begin, end).
__device__ __forceinline__ void fetch_scale(uint8_t* dst, const uint16_t* S, const uint16_t* begin,
                                            const uint16_t* end) {
    const uint8_t* wd = reinterpret_cast<const uint8_t*>(reinterpret_cast<uintptr_t>(S) & ~(uintptr_t)3);
    if (wd >= reinterpret_cast<const uint8_t*>(begin) && wd + 4 <= reinterpret_cast<const uint8_t*>(end))
        cp_async4(dst, wd);
    else
        *reinterpret_cast<uint16_t*>(dst + (reinterpret_cast<uintptr_t>(S) & 2)) = *S;
}

// FMT 3: base-3 codes; FMT 2: the 2-bit format (a stage's 64 codes are the 16
// bytes at the 16-byte-aligned offset G/4 * g + 16 * sub of the row).
template <int NT, int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemm_stream_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                                  const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem<NT>& sm = *reinterpret_cast<Smem<NT>*>(smem_raw + ((1024 - (s32(smem_raw) & 1023)) & 1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = p.K / BK;
    const int my_tiles = (p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int total = my_tiles * nk;  // stages of this CTA
    constexpr uint32_t kCols = kTmemCols<NT, FMT>, ACC = kAccCols<NT>, SLOT = kSlotCols<FMT>;
    volatile int* abort_flag = &sm.abort_flag;
    const uint64_t lim = p.wc.limit_ns;

    // Dependent launches may start now: only the X loads below wait for the
    // preceding kernel (codes and scales are weights, see tq_gemv's ordering
    // rule); every Y store follows MMAs that consumed X.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (FMT == 3) fill_digit_selector_lut4_lanes(sm.lut, threadIdx.x, kThreads);
    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(&sm.full_x[st], 1);
            mbar_init(&sm.full_w[st], kGroupWarps);
            mbar_init(&sm.empty[st], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], 4);
        }
        mbar_init(&sm.done, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s32(&sm.tmem_base)),
                     "r"(kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            asm volatile("griddepcontrol.wait;" ::: "memory");  // X comes from the preceding kernel
            int issued = 0;
            for (int i = 0; i < total; ++i) {
                const int kb = i % nk, st = i % STAGES, use = i / STAGES;
                if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag, lim)) break;
                if (!(p.wc.withhold_x && i == 0)) {  // test hook: the first load left out
                    mbar_arrive_expect_tx(&sm.full_x[st], NT * 128);
                    tma_load_2d(sm.x[st], &tmap_x, kb * BK, 0, &sm.full_x[st]);
                }
                ++issued;
            }
            // loads still in flight after an abort must land before the CTA exits
            for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
                const int st = i % STAGES, use = i / STAGES;
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sm.full_x[st], use & 1) && globaltimer() - t0 < lim) {
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = instr_desc(WM, NT);
            int i = 0;
            bool ok = true;
            for (int j = 0; j < my_tiles && ok; ++j) {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait(&sm.tempty[buf], ((j >> 1) - 1) & 1, abort_flag, lim)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * NT);
                for (int kb = 0; kb < nk; ++kb, ++i) {
                    const int st = i % STAGES, use = i / STAGES;
                    if (!mbar_wait(&sm.full_x[st], use & 1, abort_flag, lim) ||
                        !mbar_wait(&sm.full_w[st], use & 1, abort_flag, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = tmem + ACC + SLOT * (uint32_t)st, b0 = s32(sm.x[st]);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        mma_bf16_ts(d, a0 + 8u * k, smem_desc_sw128(b0 + 32 * k), idesc, (kb > 0 || k > 0) ? 1u : 0u);
                        if (FMT == 4)  // the lo terms, 32 columns on
                            mma_bf16_ts(d, a0 + 32u + 8u * k, smem_desc_sw128(b0 + 32 * k), idesc, 1u);
                    }
                    mma_commit(&sm.empty[st]);
                }
                if (ok) mma_commit(&sm.tfull[buf]);
            }
            mma_commit(&sm.done);
        }
    } else if (warp >= kDecWarp0 && warp < kEpiWarp0) {
        const int grp = (warp - kDecWarp0) >> 2;              // stages grp, grp + 2, ...
        const int t = ((warp - kDecWarp0) & 3) * 32 + lane;  // W row of the tile = tensor-memory lane
        const uint32_t trow = tmem + ((uint32_t)(t & ~31) << 16) + ACC;
        const int SPG = p.G / BK;                             // stages per group
        // stage position (tile iteration j, group g, part sub of the group),
        // advanced by two stages at a time without divisions
        struct Pos {
            int j, g, sub;
        };
        auto advance = [&](Pos& q) {
            q.sub += 2;
            while (q.sub >= SPG) {
                q.sub -= SPG;
                if (++q.g == p.ng) {
                    q.g = 0;
                    ++q.j;
                }
            }
        };
        auto row_of = [&](const Pos& q) {
            const int64_t n = ((int64_t)blockIdx.x + (int64_t)q.j * gridDim.x) * WM + t;
            return n < p.N ? n : p.N - 1;  // rows past the end decode a real row; never stored
        };
        Pos pd{0, 0, 0}, pi{0, 0, 0};  // decode position, prefetch position
        if (grp) {                      // group 1 starts at stage 1
            pd.sub = pi.sub = -1;
            advance(pd);
            pi = pd;
        }
        auto issue = [&](int s) {
            if (grp + 2 * s < total) {
                const int64_t n = row_of(pi);
                const int q_lo = FMT == 3 ? (BK * pi.sub) / 5 : (FMT == 2 ? (BK * pi.sub) / 4 : (BK * pi.sub) / 2);
                uint8_t* slot = sm.win[grp][s % CR] + t * WIN;
                fetch_window(slot, p.codes + n * p.row_bytes + (int64_t)pi.g * p.B + q_lo, p.codes, p.codes_end);
                fetch_scale(slot + 32, p.scales + n * p.ng + pi.g, p.scales, p.scales_end);
                if (FMT == 4) fetch_scale(slot + 36, p.biases + n * p.ng + pi.g, p.biases, p.biases_end);
                advance(pi);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
#pragma unroll 1
        for (int s = 0; s < CR - 1; ++s) issue(s);
        for (int s = 0; grp + 2 * s < total; ++s) {
            issue(s + CR - 1);  // its slot held own stage s - 1, decoded already
            asm volatile("cp.async.wait_group %0;" ::"n"(CR - 1) : "memory");
            const int i = grp + 2 * s, st = i % STAGES, use = i / STAGES;
            if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag, lim)) break;
            const int64_t n = row_of(pd);
            const int c0 = BK * pd.sub, q_lo = FMT == 3 ? c0 / 5 : (FMT == 2 ? c0 / 4 : c0 / 2);
            const uintptr_t A = reinterpret_cast<uintptr_t>(p.codes + n * p.row_bytes + (int64_t)pd.g * p.B + q_lo);
            const uintptr_t S = reinterpret_cast<uintptr_t>(p.scales + n * p.ng + pd.g);
            const uint8_t* slot = sm.win[grp][s % CR] + t * WIN;
            const uint8_t* cb = slot + (A & 15);
            const uint32_t sc = *reinterpret_cast<const uint16_t*>(slot + 32 + (S & 2));
            uint32_t wv[32];
            auto put = [&](int k, uint4 v) {
                wv[4 * k] = v.x;
                wv[4 * k + 1] = v.y;
                wv[4 * k + 2] = v.z;
                wv[4 * k + 3] = v.w;
            };
            if constexpr (FMT == 4) {  // codes 16-byte aligned: the window is the stage's 32 bytes
                const uint4 v0 = *reinterpret_cast<const uint4*>(slot), v1 = *reinterpret_cast<const uint4*>(slot + 16);
                const uint32_t wd[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                const uintptr_t Bi = reinterpret_cast<uintptr_t>(p.biases + n * p.ng + pd.g);
                const uint32_t bi = *reinterpret_cast<const uint16_t*>(slot + 36 + (Bi & 2));
                const float s_ = __uint_as_float(sc << 16), b_ = __uint_as_float(bi << 16);
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // columns 32 h .. 32 h + 31
                    uint32_t hv[16], lv[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {  // columns 32 h + 2 j, + 1: byte j % 4 of word 4 h + j / 4
                        const uint32_t by = wd[4 * h + (j >> 2)] >> (8 * (j & 3));
                        const float w0 = fmaf((float)(by & 0xFu), s_, b_), w1 = fmaf((float)((by >> 4) & 0xFu), s_, b_);
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(w0, w1);
                        const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h2);
                        const __nv_bfloat162 l2 = __floats2bfloat162_rn(w0 - __uint_as_float(hb << 16),
                                                                        w1 - __uint_as_float(hb & 0xFFFF0000u));
                        hv[j] = hb;
                        lv[j] = *reinterpret_cast<const uint32_t*>(&l2);
                    }
                    tmem_st16(trow + SLOT * (uint32_t)st + 16u * h, hv);
                    tmem_st16(trow + SLOT * (uint32_t)st + 32u + 16u * h, lv);
                }
            } else if constexpr (FMT == 2) {  // codes 4-byte aligned: cb is a word boundary of the window
                const uint32_t* cw = reinterpret_cast<const uint32_t*>(cb);
                const uint32_t wd[4] = {cw[0], cw[1], cw[2], cw[3]};
                decode_stage64_2bit_to(wd, sc, put);
            } else {
                uint32_t bytes[14];
#pragma unroll
                for (int b = 0; b < 14; ++b) bytes[b] = cb[b];
                const int ql = p.B - 1 - q_lo;  // the group's last byte, relative to cb
                decode_stage64_to<32>(sm.lut + (t & 31), bytes, c0 - 5 * q_lo, ql < 14, ql < 14 ? cb[ql] : 0u,
                                      p.pad_base, p.pad_span, sc, put);
            }
            if constexpr (FMT != 4) tmem_st32(trow + SLOT * (uint32_t)st, wv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.full_w[st]);
            advance(pd);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp >= kEpiWarp0) {
        const int q = warp & 3;  // TMEM lanes 32q .. 32q+31 = W rows of the tile
        uint32_t err_acc = 0;
        for (int j = 0; j < my_tiles; ++j) {
            const int buf = j & 1;
            if (!mbar_wait(&sm.tfull[buf], (j >> 1) & 1, abort_flag, lim)) break;
            tc_fence_after();
            uint32_t v[NT];
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * NT);
            if (NT == 16) {
                tmem_ld16(ta, reinterpret_cast<uint32_t (&)[16]>(v));
            } else {
#pragma unroll
                for (int h = 0; h < NT / 32; ++h) tmem_ld32(ta + 32u * h, *reinterpret_cast<uint32_t (*)[32]>(&v[32 * h]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tempty[buf]);
            const int64_t n = ((int64_t)blockIdx.x + (int64_t)j * gridDim.x) * WM + 32 * q + lane;
            if (n < p.N) {
                if (FMT != 4 && __uint_as_float(v[0]) != __uint_as_float(v[0]))  // NaN for the first token: rescan the row
                    err_acc |= FMT == 3 ? scan_row_errors(p.codes + n * p.row_bytes, p.scales + n * p.ng, p.ng, p.G, p.B)
                                        : scan_row_errors2(p.codes + n * p.row_bytes, p.scales + n * p.ng, p.ng, p.G);
#pragma unroll
                for (int m = 0; m < NT; ++m) {
                    if (m < p.M) {
                        const int64_t o = (int64_t)m * p.N + n;
                        if (p.y_bf16) reinterpret_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(__uint_as_float(v[m]));
                        else reinterpret_cast<float*>(p.Y)[o] = __uint_as_float(v[m]);
                    }
                }
            }
        }
        if (err_acc && p.d_err) atomicOr(p.d_err, err_acc);
    }

    // ---------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && lane == 0 && *abort_flag) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&sm.done, 0) && globaltimer() - t0 < lim) {
        }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 2)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
    if (threadIdx.x == 0 && *abort_flag && p.d_err) atomicOr(p.d_err, TQ_DERR_TIMEOUT);
}

template <int NT, int FMT>
static cudaError_t launch_nt(const CUtensorMap& tx, const Params& p, int grid, cudaStream_t stream) {
    auto kern = gemm_stream_kernel<NT, FMT>;
    const size_t smem = sizeof(Smem<NT>) + 1024;
    static SmemAttr smem_attr;
    if (cudaError_t e = smem_attr.ensure(kern, (int)smem)) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tx, p);
}

}  // namespace stream

// Covered shapes: 1 <= M <= 64, K % 64 == 0, G % 64 == 0.  Otherwise
// *handled is left false and nothing is launched.
cudaError_t launch_gemm_stream(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                               int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                               cudaStream_t stream, int sm_count, bool* handled, int fmt, const uint16_t* biases) {
    using namespace stream;
    *handled = false;
    if (M < 1 || M > 64 || K % BK != 0 || G % 64 != 0 || N < 1 || K > (1 << 30)) return cudaSuccess;
    // W4A16: a stage's 32 code bytes must be one 16-byte-aligned window
    if (fmt == 4 && (reinterpret_cast<uintptr_t>(codes) & 15)) return cudaSuccess;
    const int64_t tiles = (N + WM - 1) / WM;
    if (tiles > 0x7FFFFFFF / (K / BK)) return cudaSuccess;
    const int B = fmt == 3 ? bytes_per_group(G) : (fmt == 2 ? G / 4 : G / 2);
    const int NT = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    CUtensorMap tx;
    if (!encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<uint16_t*>(X), (uint64_t)K, (uint64_t)M,
                        (uint64_t)K * 2, BK, (uint32_t)NT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    Params p{};
    p.wc = tc::wait_cfg_from_env();
    p.row_bytes = (K / G) * B;
    p.codes = codes;
    p.codes_end = codes + N * p.row_bytes;
    p.scales = scales;
    p.scales_end = scales + N * (K / G);
    p.biases = biases;
    p.biases_end = biases ? biases + N * (K / G) : nullptr;
    p.Y = Y;
    p.d_err = d_err;
    p.M = M;
    p.N = N;
    p.K = (int)K;
    p.G = G;
    p.B = B;
    p.ng = (int)(K / G);
    p.tiles = (int)tiles;
    p.y_bf16 = y_bf16;
    padding_range(G, p.pad_base, p.pad_span);
    const int grid = (int)(tiles < sm_count ? tiles : sm_count);
    cudaError_t e;
    if (fmt == 4) {
        if (NT == 16) e = launch_nt<16, 4>(tx, p, grid, stream);
        else if (NT == 32) e = launch_nt<32, 4>(tx, p, grid, stream);
        else e = launch_nt<64, 4>(tx, p, grid, stream);
    } else if (fmt == 2) {
        if (NT == 16) e = launch_nt<16, 2>(tx, p, grid, stream);
        else if (NT == 32) e = launch_nt<32, 2>(tx, p, grid, stream);
        else e = launch_nt<64, 2>(tx, p, grid, stream);
    } else {
        if (NT == 16) e = launch_nt<16, 3>(tx, p, grid, stream);
        else if (NT == 32) e = launch_nt<32, 3>(tx, p, grid, stream);
        else e = launch_nt<64, 3>(tx, p, grid, stream);
    }
    if (e == cudaSuccess) *handled = true;
    return e;
}

}  // namespace tq
