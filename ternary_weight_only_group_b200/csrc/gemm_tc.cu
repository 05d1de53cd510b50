// gemm_tc.cu -- prefill GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Y[M][N] = X[M][K] . What[N][K]^T with What = t * RNE_bf16(scale) decoded on
// chip from the ternary codes ("precisit/pack-unpack-run", codec.py: base-3
// bytes, fp16 group scales; tiny-llm "Week 2 Day 3: Quantize the Model",
// "Mathematical Formulation": C = A B^T, products accumulated in float).
//
// One CTA computes a 128 x 256 tile of Y (BM rows of X, BN rows of W):
//   warp 0      TMA producer: X tiles (128 x 64 bf16, 128-byte swizzle) into
//               a 4-stage ring, completion through mbarrier transaction counts;
//   warp 1      MMA issuer: one thread issues tcgen05.mma kind::f16
//               (128 x 256 x 16, bf16 in, fp32 accumulators in tensor memory)
//               and tcgen05.commit releases each stage when its MMAs finish;
//   warp 2      allocates / frees the 256 tensor-memory columns;
//   warps 4-11  decoders: each thread owns one W row of the tile and writes
//               its 64 decoded bf16 weights per stage straight into the
//               swizzled K-major layout the MMA descriptor expects;
//   warps 4-7   epilogue: tcgen05.ld of the accumulator quadrant, bf16 or
//               fp32 stores.
// Decoding: a per-CTA table maps each code byte to the PRMT byte selectors of
// its five weights; the selectors of a stage's 14 bytes are packed into a
// stream, shifted to the stage's first column, and one PRMT per weight pair
// picks the bf16 values among {-s, 0, +s, NaN}.  Each decoder prefetches the
// next stage's scale (and, without TMA, its code bytes).  Invalid bytes,
// non-canonical padding and bad scales decode to NaN (the row's outputs are
// then NaN, as the decoder defines); the W rows behind NaN outputs of the
// first X row are rescanned for the error bits.
// Every mbarrier wait is bounded by a %globaltimer deadline; a timeout sets
// TQ_DERR_TIMEOUT, stops issuing work, drains what is in flight, frees tensor
// memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include "tc_common.cuh"

namespace tq {

namespace gemm {

using namespace tc;

constexpr int BM = 256, BN = 256, BK = 64, STAGES = 3;
constexpr int UM = 128;                     // rows of X per MMA (two MMAs per k-step)
constexpr int kThreads = 384;
constexpr int kDecodeWarp0 = 4, kDecodeWarps = 8;
constexpr uint32_t kTmemCols = 512;         // two 128 x 256 fp32 accumulators
constexpr uint32_t A_SUB = UM * BK * 2;     // 16 KB: one 128-row X subtile
constexpr uint32_t B_STAGE = BN * BK * 2;   // 32 KB: decoded W tile
constexpr uint32_t C_ROW = 32;              // code bytes fetched per W row and stage
constexpr uint32_t C_STAGE = BN * C_ROW;    // 8 KB

struct Smem {
    uint8_t a[STAGES][2][A_SUB];     // X subtiles, 1024-byte aligned
    uint8_t b[STAGES][B_STAGE];      // decoded W tiles
    uint8_t c[STAGES][C_STAGE];      // packed code bytes of the stage (TMA mode)
    uint32_t lut[256];                // byte -> PRMT selectors of its digits 0..3
    uint64_t full_a[STAGES], full_c[STAGES], full_b[STAGES], empty[STAGES], done;
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    const uint8_t* codes;
    const uint16_t* scales;
    const uint16_t* biases;  // W4A16 only
    void* Y;
    uint32_t* d_err;
    int64_t M, N;
    int K, G, B, ng;
    int64_t row_bytes;
    int n_tiles;
    int y_bf16;
    uint32_t pad_base, pad_span;  // canonical range of a group's last code byte
    WaitCfg wc;                   // wait bound and the withheld-load test hook
    int y_vec;  // Y rows allow 16-byte vector stores (base aligned, N a multiple of 16 bytes)
};

// TBN: W rows per tile (256, or 224 when that leaves a fuller last wave);
// buffers and tensor memory are laid out for 256.
// FMT 3: base-3 codes; FMT 2: the 2-bit format (a stage's 64 codes are 16
// whole bytes at a 16-byte boundary of the row); FMT 4: the W4A16 affine
// format (TBN = 128).  A W4 weight w = q * s + b (one fp32 FMA) is held as
// two bf16 tiles, hi = RNE_bf16(w) and lo = RNE_bf16(w - hi), which share
// the 32 KB W buffer of a stage; each k-step issues the MMA of both into the
// same accumulator, so the products carry w to about 2^-17 relative (one
// bf16 tile alone would carry only 2^-9).  Two threads decode a row, 32
// columns each.
template <bool CODES_TMA, int TBN, int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                              const __grid_constant__ CUtensorMap tmap_c,
                                                              const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw + ((1024 - (s32(smem_raw) & 1023)) & 1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tile = blockIdx.x / p.n_tiles, n_tile = blockIdx.x % p.n_tiles;
    const int64_t m0 = (int64_t)m_tile * BM, n0 = (int64_t)n_tile * TBN;
    const int nk = p.K / BK;
    volatile int* abort_flag = &sm.abort_flag;
    const uint64_t lim = p.wc.limit_ns;

    if (FMT == 3) fill_digit_selector_lut4(sm.lut, threadIdx.x, kThreads);
    static_assert(FMT != 4 || TBN == 128, "W4 tiles are 128 rows (hi and lo share the W buffer)");
    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) {
            mbar_init(&sm.full_a[st], 1);
            mbar_init(&sm.full_c[st], 1);
            mbar_init(&sm.full_b[st], kDecodeWarps);
            mbar_init(&sm.empty[st], 1);
        }
        mbar_init(&sm.done, 1);
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s32(&sm.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // first code byte of stage kb inside its row, and the 16-byte-aligned TMA window start
    auto stage_geom = [&](int kb, int& g, int& c0, int& q_lo) {
        const int k0 = kb * BK;
        g = k0 / p.G;
        c0 = k0 - g * p.G;
        q_lo = FMT == 3 ? c0 / 5 : (FMT == 2 ? c0 / 4 : c0 / 2);
    };

    if (warp == 0) {
        // ---------------- TMA producer: X subtiles (and the stage's code window)
        int issued = 0;
        if (lane == 0) {
            for (int kb = 0; kb < nk; ++kb) {
                const int st = kb % STAGES, use = kb / STAGES;
                if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag, lim)) break;
                if (!(p.wc.withhold_x && kb == 0)) {  // test hook: the first load left out
                    mbar_arrive_expect_tx(&sm.full_a[st], 2 * A_SUB);
                    tma_load_2d(sm.a[st][0], &tmap_x, kb * BK, (int)m0, &sm.full_a[st]);
                    tma_load_2d(sm.a[st][1], &tmap_x, kb * BK, (int)(m0 + UM), &sm.full_a[st]);
                }
                if (CODES_TMA) {
                    int g, c0, q_lo;
                    stage_geom(kb, g, c0, q_lo);
                    const int gb = g * p.B + q_lo;
                    mbar_arrive_expect_tx(&sm.full_c[st], (uint32_t)TBN * C_ROW);  // the TMA box is TBN rows
                    tma_load_2d(sm.c[st], &tmap_c, gb & ~15, (int)n0, &sm.full_c[st]);
                }
                ++issued;
            }
            // Drain: every issued load must land before the CTA can exit.
            for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb) {
                const int st = kb % STAGES, use = kb / STAGES;
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sm.full_a[st], use & 1) && globaltimer() - t0 < lim) {
                }
                if (CODES_TMA)
                    while (!mbar_try_wait(&sm.full_c[st], use & 1) && globaltimer() - t0 < lim) {
                    }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: two 128 x 256 x 16 MMAs per k-step
        if (lane == 0) {
            const uint32_t idesc = instr_desc(UM, TBN);
            for (int kb = 0; kb < nk; ++kb) {
                const int st = kb % STAGES, use = kb / STAGES;
                if (!mbar_wait(&sm.full_a[st], use & 1, abort_flag, lim)) break;
                if (!mbar_wait(&sm.full_b[st], use & 1, abort_flag, lim)) break;
                tc_fence_after();
                const uint32_t b0 = s32(sm.b[st]);
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    const uint32_t a0 = s32(sm.a[st][sub]);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        mma_bf16(tmem + (uint32_t)(sub * BN), smem_desc_sw128(a0 + 32 * k),
                                 smem_desc_sw128(b0 + 32 * k), idesc, (kb > 0 || k > 0) ? 1u : 0u);
                        if (FMT == 4)  // the lo tile, 128 rows after hi
                            mma_bf16(tmem + (uint32_t)(sub * BN), smem_desc_sw128(a0 + 32 * k),
                                     smem_desc_sw128(b0 + TBN * 128 + 32 * k), idesc, 1u);
                    }
                }
                mma_commit(&sm.empty[st]);  // stage free once these MMAs have read it
            }
            mma_commit(&sm.done);  // all issued MMAs complete -> accumulators ready
        }
    } else if (warp >= kDecodeWarp0) {
        // ---------------- decoders: thread -> one W row of the tile
        const int t = threadIdx.x - kDecodeWarp0 * 32;  // 0..255
        const int64_t n = n0 + (FMT == 4 ? (t & (TBN - 1)) : t);  // W4: two threads per row
        const bool row_ok = n < p.N;
        const uint8_t* crow = p.codes + (row_ok ? n : 0) * p.row_bytes;
        const uint16_t* srow = p.scales + (row_ok ? n : 0) * p.ng;
        const uint16_t* brow = FMT == 4 ? p.biases + (row_ok ? n : 0) * p.ng : nullptr;
        const uint8_t* w4row = crow;
        auto load_global = [&](int kb, uint32_t (&bytes)[14]) {  // code bytes of a stage, by loads
            int g, c0, q_lo;
            stage_geom(kb, g, c0, q_lo);
            const uint8_t* cb = crow + (int64_t)g * p.B;
#pragma unroll
            for (int i = 0; i < 14; ++i) bytes[i] = (q_lo + i < p.B) ? (uint32_t)__ldg(cb + q_lo + i) : kZeroByte;
        };
        uint32_t nxt[14];
        if (!CODES_TMA && FMT == 3) load_global(0, nxt);
        uint32_t sc_nxt = __ldg(srow);  // scale of stage 0 (group 0)
        uint32_t bi_nxt = FMT == 4 ? __ldg(brow) : 0u;
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % STAGES, use = kb / STAGES;
            int g, c0, q_lo;
            stage_geom(kb, g, c0, q_lo);
            const uint32_t sc = sc_nxt;
            if (kb + 1 < nk) sc_nxt = __ldg(srow + ((kb + 1) * BK) / p.G);  // next stage's scale in flight
            const uint32_t bi = bi_nxt;
            if (FMT == 4 && kb + 1 < nk) bi_nxt = __ldg(brow + ((kb + 1) * BK) / p.G);
            if constexpr (FMT == 4) {
                // thread -> row t % 128, columns 32 (t / 128) .. + 31 of the stage
                const int r = t & (TBN - 1), hh = t / TBN;
                uint32_t wd[4];
                if (CODES_TMA) {
                    if (!mbar_wait(&sm.full_c[st], use & 1, abort_flag, lim)) break;
                    const uint4 v = *reinterpret_cast<const uint4*>(sm.c[st] + r * C_ROW + 16 * hh);
                    wd[0] = v.x, wd[1] = v.y, wd[2] = v.z, wd[3] = v.w;
                } else {
                    if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag, lim)) break;
                    const uint32_t* cw = reinterpret_cast<const uint32_t*>(w4row + 32 * kb + 16 * hh);
#pragma unroll
                    for (int i = 0; i < 4; ++i) wd[i] = __ldg(cw + i);
                }
                const float s = __uint_as_float(sc << 16), b = __uint_as_float(bi << 16);
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {  // columns 2j, 2j+1: nibbles of word j / 4
                    const uint32_t wv = wd[j >> 2] >> (8 * (j & 3));
                    const float q0 = __uint_as_float(0x4B000000u | (wv & 0xFu)) - 8388608.f;
                    const float q1 = __uint_as_float(0x4B000000u | ((wv >> 4) & 0xFu)) - 8388608.f;
                    const float w0 = fmaf(q0, s, b), w1 = fmaf(q1, s, b);
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(w0, w1);
                    const uint32_t hv = *reinterpret_cast<const uint32_t*>(&h2);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(w0 - __uint_as_float(hv << 16),
                                                                    w1 - __uint_as_float(hv & 0xFFFF0000u));
                    hi[j] = hv;
                    lo[j] = *reinterpret_cast<const uint32_t*>(&l2);
                }
                uint8_t* rh = sm.b[st] + r * 128;
                uint8_t* rl = sm.b[st] + TBN * 128 + r * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int ch = ((4 * hh + c) ^ (r & 7)) << 4;
                    *reinterpret_cast<uint4*>(rh + ch) = make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                    *reinterpret_cast<uint4*>(rl + ch) = make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                }
            } else if constexpr (FMT == 2) {
                uint32_t wd[4];
                if (CODES_TMA) {
                    if (!mbar_wait(&sm.full_c[st], use & 1, abort_flag, lim)) break;
                    const uint4 v = *reinterpret_cast<const uint4*>(sm.c[st] + t * C_ROW);
                    wd[0] = v.x, wd[1] = v.y, wd[2] = v.z, wd[3] = v.w;
                } else {
                    if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag, lim)) break;
                    const uint32_t* cw = reinterpret_cast<const uint32_t*>(crow + (int64_t)g * p.B + q_lo);
#pragma unroll
                    for (int i = 0; i < 4; ++i) wd[i] = __ldg(cw + i);
                }
                if (t < TBN) decode_stage64_2bit(wd, sc, sm.b[st] + t * 128, t & 7);
            } else {
            const int ql = p.B - 1 - q_lo;  // the group's last byte relative to q_lo
            uint32_t bytes[14], lastb = 0;
            if (CODES_TMA) {
                if (!mbar_wait(&sm.full_c[st], use & 1, abort_flag, lim)) break;
                const int gb = g * p.B + q_lo;
                const uint8_t* win = sm.c[st] + t * C_ROW;
                window_bytes(win, gb & 15, bytes);
                if (ql < 14) lastb = win[(gb & 15) + ql];
            } else {
#pragma unroll
                for (int i = 0; i < 14; ++i) bytes[i] = nxt[i];
                if (kb + 1 < nk) load_global(kb + 1, nxt);  // next stage's bytes in flight
                if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag, lim)) break;
                if (ql < 14) lastb = __ldg(crow + (int64_t)g * p.B + p.B - 1);
            }
            if (t < TBN)
                decode_stage64(sm.lut, bytes, c0 - 5 * q_lo, ql < 14, lastb, p.pad_base, p.pad_span, sc,
                               sm.b[st] + t * 128, t & 7);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.full_b[st]);
        }
        // ---------------- epilogue: warps 4..7 read their accumulator quadrant
        if (warp < kDecodeWarp0 + 4) {
            const int q = warp - kDecodeWarp0;  // TMEM lanes 32q .. 32q+31
            uint32_t err_acc = 0;
            const bool ok = mbar_wait(&sm.done, 0, abort_flag, lim);
            tc_fence_after();
            if (ok && !*abort_flag) {  // after a wait gave up, Y is left as it was
                for (int sub = 0; sub < 2; ++sub) {
                    const int64_t m = m0 + sub * UM + 32 * q + lane;
                    for (int c = 0; c < TBN / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(sub * BN + 32 * c), r);
                        const int64_t nb = n0 + 32 * c;
                        if (m < p.M && nb < p.N) {
                            const int cnt = (int)(p.N - nb < 32 ? p.N - nb : 32);
                            if (m == 0 && FMT != 4) {  // a NaN output of the first X row: rescan that W row's groups
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (j < cnt && __uint_as_float(r[j]) != __uint_as_float(r[j]))
                                        err_acc |= FMT == 3 ? scan_row_errors(p.codes + (nb + j) * p.row_bytes,
                                                                              p.scales + (nb + j) * p.ng, p.ng, p.G, p.B)
                                                            : scan_row_errors2(p.codes + (nb + j) * p.row_bytes,
                                                                               p.scales + (nb + j) * p.ng, p.ng, p.G);
                            }
                            if (p.y_bf16) {
                                __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(p.Y) + m * p.N + nb;
                                if (cnt == 32 && p.y_vec) {
#pragma unroll
                                    for (int v = 0; v < 4; ++v) {
                                        uint32_t w[4];
#pragma unroll
                                        for (int h = 0; h < 4; ++h) {
                                            const __nv_bfloat162 b2 =
                                                __floats2bfloat162_rn(__uint_as_float(r[8 * v + 2 * h]),
                                                                      __uint_as_float(r[8 * v + 2 * h + 1]));
                                            w[h] = *reinterpret_cast<const uint32_t*>(&b2);
                                        }
                                        reinterpret_cast<uint4*>(y)[v] = make_uint4(w[0], w[1], w[2], w[3]);
                                    }
                                } else {
#pragma unroll
                                    for (int j = 0; j < 32; ++j)
                                        if (j < cnt) y[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
                                }
                            } else {
                                float* y = reinterpret_cast<float*>(p.Y) + m * p.N + nb;
                                if (cnt == 32 && p.y_vec) {
#pragma unroll
                                    for (int v = 0; v < 8; ++v)
                                        reinterpret_cast<float4*>(y)[v] =
                                            make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                        __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
                                } else {
#pragma unroll
                                    for (int j = 0; j < 32; ++j)
                                        if (j < cnt) y[j] = __uint_as_float(r[j]);
                                }
                            }
                        }
                    }
                }
            }
            if (err_acc && p.d_err) atomicOr(p.d_err, err_acc);
        }
    }

    // ---------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && lane == 0 && *abort_flag) {
        // The commit after the issue loop tracks every MMA this CTA issued:
        // wait for it (bounded) before tensor memory is freed.
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&sm.done, 0) && globaltimer() - t0 < lim) {
        }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 2)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    if (threadIdx.x == 0 && *abort_flag && p.d_err) atomicOr(p.d_err, TQ_DERR_TIMEOUT);
}

// ------------------------------------------------------------------ host

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_impl() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

}  // namespace gemm

namespace tc {
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, void* base, uint64_t dim0, uint64_t dim1,
                    uint64_t stride1_bytes, uint32_t box0, uint32_t box1, CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = gemm::encode_fn_impl();
    if (!enc) return false;
    std::memset(map, 0, sizeof(*map));
    const cuuint64_t gdim[2] = {(cuuint64_t)dim0, (cuuint64_t)dim1};
    const cuuint64_t gstride[1] = {(cuuint64_t)stride1_bytes};
    const cuuint32_t box[2] = {box0, box1};
    const cuuint32_t estride[2] = {1, 1};
    return enc(map, dtype, 2, base, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace tc

size_t gemm_smem_bytes() { return sizeof(gemm::Smem) + 1024; }

cudaError_t launch_gemm_tc(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales, int64_t N,
                           int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err, cudaStream_t stream,
                           int sm_count, bool* handled, int fmt, const uint16_t* biases) {
    using namespace gemm;
    *handled = false;
    // Shapes this kernel covers: K a multiple of the 64-column stage, G a
    // multiple of 64 (a stage never crosses a group).
    if (K % BK != 0 || G % 64 != 0 || M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (1 << 30))
        return cudaSuccess;
    const int B = fmt == 3 ? bytes_per_group(G) : (fmt == 2 ? G / 4 : G / 2);
    const int64_t row_bytes = (int64_t)(K / G) * B;
    CUtensorMap tmap_x, tmap_c;
    std::memset(&tmap_c, 0, sizeof(tmap_c));
    if (!encode_tmap_2d(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<uint16_t*>(X), (uint64_t)K,
                        (uint64_t)M, (uint64_t)K * 2, BK, UM, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // Codes by TMA when their rows are 16-byte multiples and the base is 16-byte aligned.
    const bool codes_tma = (row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(codes) & 15) == 0);
    // W rows per tile: 256, or 224 when the grid then ends in a fuller wave
    // (fewer waves x tile width; every CTA runs one tile, one CTA per SM)
    const int64_t m_tiles = (M + BM - 1) / BM;
    auto cost = [&](int bn) {
        const int64_t tiles = m_tiles * ((N + bn - 1) / bn);
        return ((tiles + sm_count - 1) / sm_count) * bn;
    };
    const int tbn = fmt == 4 ? 128 : (cost(224) < cost(256) ? 224 : 256);
    if (codes_tma && !encode_tmap_2d(&tmap_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<uint8_t*>(codes),
                                     (uint64_t)row_bytes, (uint64_t)N, (uint64_t)row_bytes, C_ROW, (uint32_t)tbn,
                                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    Params p{};
    p.wc = tc::wait_cfg_from_env();
    p.codes = codes;
    p.scales = scales;
    p.biases = biases;
    p.Y = Y;
    p.d_err = d_err;
    p.M = M;
    p.N = N;
    p.K = (int)K;
    p.G = G;
    p.B = B;
    p.ng = (int)(K / G);
    p.row_bytes = row_bytes;
    p.n_tiles = (int)((N + tbn - 1) / tbn);
    padding_range(G, p.pad_base, p.pad_span);
    p.y_bf16 = y_bf16;
    p.y_vec = ((reinterpret_cast<uintptr_t>(Y) & 15) == 0) && ((N * (y_bf16 ? 2 : 4)) % 16 == 0);
    const int64_t grid = m_tiles * p.n_tiles;
    if (grid > 0x7FFFFFFF) return cudaSuccess;
    const size_t smem = gemm_smem_bytes();
    auto kern = fmt == 4   ? (codes_tma ? gemm_tc_kernel<true, 128, 4> : gemm_tc_kernel<false, 128, 4>)
                : fmt == 2 ? (codes_tma ? (tbn == 224 ? gemm_tc_kernel<true, 224, 2> : gemm_tc_kernel<true, 256, 2>)
                                        : (tbn == 224 ? gemm_tc_kernel<false, 224, 2> : gemm_tc_kernel<false, 256, 2>))
                           : (codes_tma ? (tbn == 224 ? gemm_tc_kernel<true, 224, 3> : gemm_tc_kernel<true, 256, 3>)
                                        : (tbn == 224 ? gemm_tc_kernel<false, 224, 3> : gemm_tc_kernel<false, 256, 3>));
    static SmemAttr smem_attr[10];
    const int slot = fmt == 4 ? 8 + (codes_tma ? 1 : 0) : (fmt == 2 ? 4 : 0) + (codes_tma ? 2 : 0) + (tbn == 224 ? 1 : 0);
    if (cudaError_t e = smem_attr[slot].ensure(kern, (int)smem)) return e;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(tmap_x, tmap_c, p);
    *handled = true;
    return cudaGetLastError();
}

}  // namespace tq
