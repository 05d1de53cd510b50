// gemm_small.cu -- small-M fused matmul on the tensor cores (tcgen05, sm_100a).
//
// Same result as the decode GEMV and the prefill GEMM (tiny-llm "Week 2 Day
// 3: Quantize the Model", "Mathematical Formulation": C = A B^T with B
// reconstructed per group, float accumulation; "Tune the SIMD Schedule":
// the decode and matrix schedules are chosen by M), for 5 <= M <= 64 tokens.
// The roles of the operands are swapped so the tensor core's 128-row side is
// filled by weights:  D^T[128 W rows x NT tokens] += What[128 x 16] . X[NT x 16]^T
// with What decoded on chip straight into tensor memory (each decoder thread
// owns one W row = one tensor-memory lane and stores its 64 bf16 of a stage
// with tcgen05.st), where the MMA reads it as the A operand, and X tiles
// (NT = 16, 32 or 64 rows, zero-filled past M) loaded by TMA.  K is split
// across the CTAs of a thread-block cluster; each CTA pushes its fp32 partial
// tile into the shared memory of the rank that owns those rows (distributed
// shared memory), one cluster barrier, and the owner adds the partials in
// rank order (deterministic) and writes Y.  In a chain of launches a CTA
// decodes (up to seven stages) while the preceding kernel still runs: only
// the X loads wait for it.
//   warp 0  TMA producer (code-byte windows, then X tiles)
//   warp 1  MMA issuer (tcgen05.mma kind::f16, M=128, N=NT, A in tensor memory)
//   warp 2  tensor-memory allocation
//   warps 4-7  decoders (one W row per thread), then the epilogue
// All mbarrier waits are bounded (globaltimer deadline -> TQ_DERR_TIMEOUT).
#include <cooperative_groups.h>

#include <atomic>
#include <cstring>

#include "tc_common.cuh"

namespace cg = cooperative_groups;

namespace tq {
namespace small {

using namespace tc;

constexpr int WM = 128;  // W rows per CTA (UMMA M)
constexpr int BK = 64;
// Tensor memory: 256 columns per CTA (two CTAs per SM use all 512): the
// accumulator D in columns [0, ACC) and WSL slots of decoded W, 32 columns
// (one 128 x 64 bf16 stage) each, as the MMA's A operand.  Shared memory
// holds no decoded weights: X tiles in a ring of XS, code windows in a ring
// of CST (deep enough for a CTA's whole K slice at the shapes that take this
// kernel), so every code window is requested before the grid-dependency wait
// and every X tile right after it.
constexpr uint32_t kCols = 256;
template <int NT>
constexpr int kAcc = NT < 32 ? 32 : NT;
template <int NT>
constexpr int kWSlots = (int)(kCols - kAcc<NT>) / 32;  // 7, 7, 6
// W4A16 (FMT 4): a stage holds each weight as two bf16 terms, hi and lo, in a
// pair of 32-column slots (3 pairs)
template <int NT, int FMT>
constexpr int kWSlotsF = (int)(kCols - kAcc<NT>) / (FMT == 4 ? 64 : 32);
template <int NT>
constexpr int kXStages = NT == 64 ? 4 : 8;
constexpr int kCStages = 8;
constexpr int kThreads = 256;
constexpr int kDecodeWarp0 = 4, kDecodeWarps = 4;
constexpr uint32_t C_ROW = 32;
constexpr uint32_t C_STAGE = WM * C_ROW;   // 4 KB
constexpr int kMaxCS = 8;
// At least this much dynamic shared memory per CTA, so that no more than two
// CTAs (2 x 256 tensor-memory columns) ever share an SM.
constexpr size_t kMinSmem = 80 * 1024;

template <int NT>
struct Smem {
    static constexpr int XS = kXStages<NT>, CST = kCStages, WSL = kWSlots<NT>;
    uint8_t x[XS][NT * 128];      // X tiles (UMMA B): NT rows of 128 bytes, 1024-byte aligned
    uint8_t c[CST][C_STAGE];      // code-byte windows
    // partials pushed by the cluster: [rank][row of owner][token], rows NT + 4
    // floats apart, so that eight lanes storing or loading 16 bytes of eight
    // consecutive rows cover all 32 banks
    float red[WM * (NT + 4)];
    uint32_t lut[256];                // byte -> PRMT selectors of its digits 0..3
    uint64_t full_x[XS], xempty[XS], full_c[CST], cempty[CST], full_w[WSL], wempty[WSL], done;
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    const uint8_t* codes;
    int64_t row_bytes;
    const uint16_t* scales;
    const uint16_t* biases;  // W4A16 only
    void* Y;
    uint32_t* d_err;
    int64_t M, N;
    int K, G, B, ng;
    int CS;  // cluster size = split of K
    int y_bf16;
    uint32_t pad_base, pad_span;  // canonical range of a group's last code byte
    WaitCfg wc;                   // wait bound and the withheld-load test hook
};

// FMT 3: base-3 codes (five digits per byte); FMT 2: the 2-bit format (four
// codes per byte, G a multiple of 64: a stage's 64 codes are 16 whole bytes);
// FMT 4: the W4A16 affine codes (two per byte, a stage's 64 codes are 32
// bytes at a 32-byte boundary of the row), each weight w = q * s + b by one
// fp32 FMA held as hi = RNE_bf16(w) and lo = RNE_bf16(w - hi), both MMAs
// into the same accumulator.
template <int NT, bool CODES_TMA, int FMT>
__global__ void __launch_bounds__(kThreads, 2) gemm_small_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                                 const __grid_constant__ CUtensorMap tmap_c,
                                                                 const Params p) {
    constexpr int XS = kXStages<NT>, CST = kCStages, WSL = kWSlotsF<NT, FMT>;
    constexpr uint32_t ACC = kAcc<NT>, SLOT = FMT == 4 ? 64u : 32u;  // columns per stage slot
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem<NT>& sm = *reinterpret_cast<Smem<NT>*>(smem_raw + ((1024 - (s32(smem_raw) & 1023)) & 1023));
    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)(blockIdx.x / p.CS) * WM;
    const int nk = p.K / BK;
    const int kb_lo = (int)((int64_t)nk * crank / p.CS), kb_hi = (int)((int64_t)nk * (crank + 1) / p.CS);
    const int nkl = kb_hi - kb_lo;  // stages of this CTA (>= 1)
    volatile int* abort_flag = &sm.abort_flag;
    const uint64_t lim = p.wc.limit_ns;

    // Dependent launches may start now: only the X loads below wait for the
    // preceding kernel (codes and scales are weights, see tq_gemv's ordering
    // rule); every Y store follows MMAs that consumed X.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    cluster_arrive_relaxed();  // waited on before the first store into a peer's shared memory
    if (FMT == 3) fill_digit_selector_lut4(sm.lut, threadIdx.x, kThreads);
    if (threadIdx.x == 0) {
        for (int i = 0; i < XS; ++i) {
            mbar_init(&sm.full_x[i], 1);
            mbar_init(&sm.xempty[i], 1);
        }
        for (int i = 0; i < CST; ++i) {
            mbar_init(&sm.full_c[i], 1);
            mbar_init(&sm.cempty[i], kDecodeWarps);
        }
        for (int i = 0; i < WSL; ++i) {
            mbar_init(&sm.full_w[i], kDecodeWarps);
            mbar_init(&sm.wempty[i], 1);
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
    cluster_wait();  // every CTA of the cluster is running: the partial pushes below may target it
    const uint32_t tmem = sm.tmem_base;

    auto stage_geom = [&](int kb, int& g, int& c0, int& q_lo) {
        const int k0 = kb * BK;
        g = k0 / p.G;
        c0 = k0 - g * p.G;
        q_lo = FMT == 3 ? c0 / 5 : (FMT == 2 ? c0 / 4 : c0 / 2);
    };

    if (warp == 0) {
        if (lane == 0) {
            auto load_c = [&](int i) {
                int g, c0, q_lo;
                stage_geom(kb_lo + i, g, c0, q_lo);
                mbar_arrive_expect_tx(&sm.full_c[i % CST], C_STAGE);
                tma_load_2d(sm.c[i % CST], &tmap_c, (g * p.B + q_lo) & ~15, (int)n0, &sm.full_c[i % CST]);
            };
            auto load_x = [&](int i) {
                if (p.wc.withhold_x && i == 0) return;  // test hook: the first load left out
                mbar_arrive_expect_tx(&sm.full_x[i % XS], NT * 128);
                tma_load_2d(sm.x[i % XS], &tmap_x, (kb_lo + i) * BK, 0, &sm.full_x[i % XS]);
            };
            int ci = 0, xi = 0;  // code windows and X tiles issued
            if (CODES_TMA)
                for (; ci < nkl && ci < CST; ++ci) load_c(ci);
            asm volatile("griddepcontrol.wait;" ::: "memory");  // X comes from the preceding kernel
            for (; xi < nkl && xi < XS; ++xi) load_x(xi);
            for (int i = 0; i < nkl; ++i) {
                if (CODES_TMA && i >= CST) {
                    if (!mbar_wait(&sm.cempty[i % CST], (i / CST - 1) & 1, abort_flag, lim)) break;
                    load_c(i);
                    ci = i + 1;
                }
                if (i >= XS) {
                    if (!mbar_wait(&sm.xempty[i % XS], (i / XS - 1) & 1, abort_flag, lim)) break;
                    load_x(i);
                    xi = i + 1;
                }
            }
            // let every copy in flight land before the CTA can exit
            const uint64_t t0 = globaltimer();
            for (int i = (xi > XS ? xi - XS : 0); i < xi; ++i)
                while (!mbar_try_wait(&sm.full_x[i % XS], (i / XS) & 1) && globaltimer() - t0 < lim) {
                }
            for (int i = (ci > CST ? ci - CST : 0); i < ci; ++i)
                while (!mbar_try_wait(&sm.full_c[i % CST], (i / CST) & 1) && globaltimer() - t0 < lim) {
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = instr_desc(WM, NT);
            for (int i = 0; i < nkl; ++i) {
                const int st = i % WSL;
                if (!mbar_wait(&sm.full_x[i % XS], (i / XS) & 1, abort_flag, lim)) break;
                if (!mbar_wait(&sm.full_w[st], (i / WSL) & 1, abort_flag, lim)) break;
                tc_fence_after();
                const uint32_t a0 = tmem + ACC + SLOT * (uint32_t)st, b0 = s32(sm.x[i % XS]);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k) {
                    mma_bf16_ts(tmem, a0 + 8u * k, smem_desc_sw128(b0 + 32 * k), idesc, (i > 0 || k > 0) ? 1u : 0u);
                    if (FMT == 4)  // the lo terms, 32 columns on
                        mma_bf16_ts(tmem, a0 + 32u + 8u * k, smem_desc_sw128(b0 + 32 * k), idesc, 1u);
                }
                mma_commit(&sm.wempty[st]);
                mma_commit(&sm.xempty[i % XS]);
            }
            mma_commit(&sm.done);
        }
    } else if (warp >= kDecodeWarp0) {
        const int t = threadIdx.x - kDecodeWarp0 * 32;  // W row of the tile = tensor-memory lane
        const uint32_t trow = tmem + ((uint32_t)(32 * (warp - kDecodeWarp0)) << 16) + ACC;
        const int64_t n = n0 + t;
        const uint16_t* srow = p.scales + (n < p.N ? n : 0) * p.ng;
        const uint16_t* brow = FMT == 4 ? p.biases + (n < p.N ? n : 0) * p.ng : nullptr;
        const uint8_t* crow = p.codes + (n < p.N ? n : 0) * p.row_bytes;
        auto load_global = [&](int kb, uint32_t (&bytes)[14]) {
            int g, c0, q_lo;
            stage_geom(kb, g, c0, q_lo);
            const uint8_t* cb = crow + (int64_t)g * p.B;
#pragma unroll
            for (int j = 0; j < 14; ++j) bytes[j] = (q_lo + j < p.B) ? (uint32_t)__ldg(cb + q_lo + j) : kZeroByte;
        };
        uint32_t cur[14], nxt[14];
        if (!CODES_TMA && FMT == 3 && nkl > 0) load_global(kb_lo, cur);
        uint32_t sc_nxt = nkl > 0 ? __ldg(srow + (kb_lo * BK) / p.G) : 0u;
        uint32_t bi_nxt = FMT == 4 && nkl > 0 ? __ldg(brow + (kb_lo * BK) / p.G) : 0u;
        for (int i = 0; i < nkl; ++i) {
            const int kb = kb_lo + i, st = i % WSL, use = i / WSL;
            int g, c0, q_lo;
            stage_geom(kb, g, c0, q_lo);
            const uint32_t sc = sc_nxt;
            if (i + 1 < nkl) sc_nxt = __ldg(srow + ((kb + 1) * BK) / p.G);  // next stage's scale in flight
            const uint32_t bi = bi_nxt;
            if (FMT == 4 && i + 1 < nkl) bi_nxt = __ldg(brow + ((kb + 1) * BK) / p.G);
            uint32_t wv[32];
            auto put = [&](int k, uint4 v) {
                wv[4 * k] = v.x;
                wv[4 * k + 1] = v.y;
                wv[4 * k + 2] = v.z;
                wv[4 * k + 3] = v.w;
            };
            // the window's bytes are in registers: the window may be refilled
            auto release_window = [&]() {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.cempty[i % CST]);
            };
            if constexpr (FMT == 4) {
                // the stage's 32 code bytes (64 nibbles, low nibble first)
                uint32_t wd[8];
                if (CODES_TMA) {
                    if (!mbar_wait(&sm.full_c[i % CST], (i / CST) & 1, abort_flag, lim)) break;
                    const uint4* cw = reinterpret_cast<const uint4*>(sm.c[i % CST] + t * C_ROW);
                    const uint4 v0 = cw[0], v1 = cw[1];
                    wd[0] = v0.x, wd[1] = v0.y, wd[2] = v0.z, wd[3] = v0.w;
                    wd[4] = v1.x, wd[5] = v1.y, wd[6] = v1.z, wd[7] = v1.w;
                    release_window();
                } else {
                    const uint32_t* cw = reinterpret_cast<const uint32_t*>(crow + (int64_t)g * p.B + q_lo);
#pragma unroll
                    for (int j = 0; j < 8; ++j) wd[j] = __ldg(cw + j);
                }
                if (use > 0 && !mbar_wait(&sm.wempty[st], (use - 1) & 1, abort_flag, lim)) break;
                const float s = __uint_as_float(sc << 16), b = __uint_as_float(bi << 16);
#pragma unroll
                for (int h = 0; h < 2; ++h) {  // columns 32 h .. 32 h + 31
                    uint32_t hv[16], lv[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {  // columns 32 h + 2 j, + 1: byte j % 4 of word 4 h + j / 4
                        const uint32_t by = wd[4 * h + (j >> 2)] >> (8 * (j & 3));
                        const float w0 = fmaf((float)(by & 0xFu), s, b), w1 = fmaf((float)((by >> 4) & 0xFu), s, b);
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
            } else if constexpr (FMT == 2) {
                // the stage's 16 code bytes start on a 16-byte boundary of the row
                uint32_t wd[4];
                if (CODES_TMA) {
                    if (!mbar_wait(&sm.full_c[i % CST], (i / CST) & 1, abort_flag, lim)) break;
                    const uint4 v = *reinterpret_cast<const uint4*>(sm.c[i % CST] + t * C_ROW);
                    wd[0] = v.x, wd[1] = v.y, wd[2] = v.z, wd[3] = v.w;
                    release_window();
                } else {
                    const uint32_t* cw = reinterpret_cast<const uint32_t*>(crow + (int64_t)g * p.B + q_lo);
#pragma unroll
                    for (int j = 0; j < 4; ++j) wd[j] = __ldg(cw + j);
                }
                if (use > 0 && !mbar_wait(&sm.wempty[st], (use - 1) & 1, abort_flag, lim)) break;
                decode_stage64_2bit_to(wd, sc, put);
            } else {
                const int ql = p.B - 1 - q_lo;  // the group's last byte relative to q_lo
                uint32_t bytes[14], lastb = 0;
                if (CODES_TMA) {
                    if (!mbar_wait(&sm.full_c[i % CST], (i / CST) & 1, abort_flag, lim)) break;
                    const int off = (g * p.B + q_lo) & 15;
                    const uint8_t* win = sm.c[i % CST] + t * C_ROW;
                    window_bytes(win, off, bytes);
                    if (ql < 14) lastb = win[off + ql];
                    release_window();
                } else {
                    if (i + 1 < nkl) load_global(kb + 1, nxt);  // next stage's bytes in flight
#pragma unroll
                    for (int j = 0; j < 14; ++j) bytes[j] = cur[j];
                    if (ql < 14) lastb = __ldg(crow + (int64_t)g * p.B + p.B - 1);
                }
                if (use > 0 && !mbar_wait(&sm.wempty[st], (use - 1) & 1, abort_flag, lim)) break;
                decode_stage64_to<1>(sm.lut, bytes, c0 - 5 * q_lo, ql < 14, lastb, p.pad_base, p.pad_span, sc, put);
                if (!CODES_TMA) {
#pragma unroll
                    for (int j = 0; j < 14; ++j) cur[j] = nxt[j];
                }
            }
            if constexpr (FMT != 4) tmem_st32(trow + SLOT * (uint32_t)st, wv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.full_w[st]);
        }
    }

    // ---------------- epilogue: partial tile -> owner ranks -> Y
    const int RPQ = WM / p.CS;  // rows owned by each rank
    if (warp >= kDecodeWarp0) {
        const int q = warp - kDecodeWarp0;
        const int r = 32 * q + lane;  // W row of the tile = TMEM lane
        const bool ok = mbar_wait(&sm.done, 0, abort_flag, lim);
        tc_fence_after();
        uint32_t v[NT];
        if (NT == 16) {
            uint32_t (&v16)[16] = reinterpret_cast<uint32_t (&)[16]>(v);
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16), v16);
        } else {
#pragma unroll
            for (int h = 0; h < NT / 32; ++h) {
                uint32_t (&v32)[32] = *reinterpret_cast<uint32_t (*)[32]>(&v[32 * h]);
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + 32u * h, v32);
            }
        }
        if (!ok || *abort_flag) {  // a wait gave up: the partial is not defined
#pragma unroll
            for (int j = 0; j < NT; ++j) v[j] = 0x7FC00000u;
        }
        const int owner = r / RPQ;
        float* dst = cluster.map_shared_rank(sm.red, owner) + ((crank * RPQ) + (r - owner * RPQ)) * (NT + 4);
#pragma unroll
        for (int j = 0; j < NT; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                              __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
    }
    tc_fence_before();
    cluster.sync();
    tc_fence_after();
    // owner: rows [crank*RPQ, (crank+1)*RPQ) of the tile, all tokens; a thread
    // adds four tokens of one row (16-byte loads), consecutive lanes take
    // consecutive rows, so each token's stores cover consecutive outputs
    const int64_t Mv = p.M < NT ? p.M : NT;
    const int MQ = (int)((Mv + 3) / 4);
    uint32_t err_acc = 0;
    for (int i = threadIdx.x; i < RPQ * MQ; i += kThreads) {
        const int mq = i / RPQ, rr = i - mq * RPQ;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int qr = 0; qr < p.CS; ++qr) {
            const float4 v4 = *reinterpret_cast<const float4*>(&sm.red[(qr * RPQ + rr) * (NT + 4) + 4 * mq]);
            acc.x += v4.x;
            acc.y += v4.y;
            acc.z += v4.z;
            acc.w += v4.w;
        }
        const int64_t n = n0 + crank * RPQ + rr;
        if (n < p.N) {
            const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
            if (FMT != 4 && mq == 0 && acc.x != acc.x)  // NaN output of the first token: rescan that W row
                err_acc |= FMT == 3 ? scan_row_errors(p.codes + n * p.row_bytes, p.scales + n * p.ng, p.ng, p.G, p.B)
                                    : scan_row_errors2(p.codes + n * p.row_bytes, p.scales + n * p.ng, p.ng, p.G);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int64_t m = 4 * mq + t;
                if (m < Mv) {
                    const int64_t o = m * p.N + n;
                    if (p.y_bf16) reinterpret_cast<__nv_bfloat16*>(p.Y)[o] = __float2bfloat16_rn(a4[t]);
                    else reinterpret_cast<float*>(p.Y)[o] = a4[t];
                }
            }
        }
    }

    if (err_acc && p.d_err) atomicOr(p.d_err, err_acc);

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

template <int NT, bool CT, int FMT>
static cudaError_t launch_nt(const CUtensorMap& tx, const CUtensorMap& tc_, const Params& p, int tiles,
                             cudaStream_t stream) {
    auto kern = gemm_small_kernel<NT, CT, FMT>;
    const size_t smem = sizeof(Smem<NT>) + 1024 > kMinSmem ? sizeof(Smem<NT>) + 1024 : kMinSmem;
    static SmemAttr smem_attr;
    if (cudaError_t e = smem_attr.ensure(kern, (int)smem)) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * p.CS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tx, tc_, p);
}

}  // namespace small

cudaError_t launch_gemm_stream(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                               int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                               cudaStream_t stream, int sm_count, bool* handled, int fmt, const uint16_t* biases);

// Covered shapes: 1 <= M <= 64, K % 64 == 0, G % 64 == 0.  Otherwise *handled is
// left false and nothing is launched.  fmt: 3 base-3 codes, 2 the 2-bit format,
// 4 the W4A16 affine codes with `biases` (the persistent kernel needs
// 16-byte-aligned codes for them, else the shape is left unhandled).
cudaError_t launch_gemm_small(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                              int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                              cudaStream_t stream, int sm_count, bool* handled, int fmt, const uint16_t* biases) {
    using namespace small;
    *handled = false;
    const int B = fmt == 3 ? bytes_per_group(G) : (fmt == 2 ? G / 4 : G / 2);
    const int64_t row_bytes = (int64_t)(K / G) * B;
    if (M < 1 || M > 64 || K % BK != 0 || G % 64 != 0 || N > (int64_t(1) << 31) || K > (1 << 30))
        return cudaSuccess;
    // code bytes by TMA when their rows are 16-byte multiples with an aligned base, else by loads
    const bool codes_tma = row_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
    const int NT = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    CUtensorMap tx, tcm;
    if (!encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<uint16_t*>(X), (uint64_t)K, (uint64_t)M,
                        (uint64_t)K * 2, BK, (uint32_t)NT, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    std::memset(&tcm, 0, sizeof(tcm));
    if (codes_tma && !encode_tmap_2d(&tcm, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<uint8_t*>(codes),
                                     (uint64_t)row_bytes, (uint64_t)N, (uint64_t)row_bytes, C_ROW, WM,
                                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const int nk = (int)(K / BK);
    const int64_t tiles = (N + WM - 1) / WM;
    if (tiles * kMaxCS > 0x7FFFFFFF) return cudaSuccess;
    // split K so the grid covers the SMs, keeping at least two stages per CTA
    int CS = 1;
    // at most one CTA per SM: the next dependent launch finds a free slot on
    // every SM (16/32-token tiles fit twice) and decodes before its wait
    const int64_t slots = (int64_t)sm_count;
    while (CS < kMaxCS && tiles * CS * 2 <= slots && nk / (CS * 2) >= 2) CS *= 2;
    if (CS == 1)  // no K split: the persistent kernel walks the tiles
        return launch_gemm_stream(X, M, codes, scales, N, K, G, Y, y_bf16, d_err, stream, sm_count, handled, fmt,
                                  biases);
    Params p{};
    p.wc = tc::wait_cfg_from_env();
    p.codes = codes;
    p.row_bytes = row_bytes;
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
    p.CS = CS;
    p.y_bf16 = y_bf16;
    padding_range(G, p.pad_base, p.pad_span);
    cudaError_t e;
    if (fmt == 4) {
        if (codes_tma) {
            if (NT == 16) e = launch_nt<16, true, 4>(tx, tcm, p, (int)tiles, stream);
            else if (NT == 32) e = launch_nt<32, true, 4>(tx, tcm, p, (int)tiles, stream);
            else e = launch_nt<64, true, 4>(tx, tcm, p, (int)tiles, stream);
        } else {
            if (NT == 16) e = launch_nt<16, false, 4>(tx, tcm, p, (int)tiles, stream);
            else if (NT == 32) e = launch_nt<32, false, 4>(tx, tcm, p, (int)tiles, stream);
            else e = launch_nt<64, false, 4>(tx, tcm, p, (int)tiles, stream);
        }
    } else if (fmt == 2) {
        if (codes_tma) {
            if (NT == 16) e = launch_nt<16, true, 2>(tx, tcm, p, (int)tiles, stream);
            else if (NT == 32) e = launch_nt<32, true, 2>(tx, tcm, p, (int)tiles, stream);
            else e = launch_nt<64, true, 2>(tx, tcm, p, (int)tiles, stream);
        } else {
            if (NT == 16) e = launch_nt<16, false, 2>(tx, tcm, p, (int)tiles, stream);
            else if (NT == 32) e = launch_nt<32, false, 2>(tx, tcm, p, (int)tiles, stream);
            else e = launch_nt<64, false, 2>(tx, tcm, p, (int)tiles, stream);
        }
    } else if (codes_tma) {
        if (NT == 16) e = launch_nt<16, true, 3>(tx, tcm, p, (int)tiles, stream);
        else if (NT == 32) e = launch_nt<32, true, 3>(tx, tcm, p, (int)tiles, stream);
        else e = launch_nt<64, true, 3>(tx, tcm, p, (int)tiles, stream);
    } else {
        if (NT == 16) e = launch_nt<16, false, 3>(tx, tcm, p, (int)tiles, stream);
        else if (NT == 32) e = launch_nt<32, false, 3>(tx, tcm, p, (int)tiles, stream);
        else e = launch_nt<64, false, 3>(tx, tcm, p, (int)tiles, stream);
    }
    if (e == cudaSuccess) *handled = true;
    return e;
}

}  // namespace tq
