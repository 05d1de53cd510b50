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
// its five weights; one PRMT gathers the selectors of a weight pair, a second
// PRMT picks the pair's bf16 values among {+s, -s, 0, NaN}.  Invalid bytes,
// non-canonical padding and bad scales decode to NaN (the row's outputs are
// then NaN, as the decoder defines).
// Every mbarrier wait is bounded by a %globaltimer deadline; a timeout sets
// TQ_DERR_TIMEOUT, stops issuing work, drains what is in flight, frees tensor
// memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include "tq_internal.cuh"

namespace tq {

namespace gemm {

constexpr int BM = 256, BN = 256, BK = 64, STAGES = 3;
constexpr int UM = 128;                     // rows of X per MMA (two MMAs per k-step)
constexpr int kThreads = 384;
constexpr int kDecodeWarp0 = 4, kDecodeWarps = 8;
constexpr uint32_t kTmemCols = 512;         // two 128 x 256 fp32 accumulators
constexpr uint32_t A_SUB = UM * BK * 2;     // 16 KB: one 128-row X subtile
constexpr uint32_t B_STAGE = BN * BK * 2;   // 32 KB: decoded W tile
constexpr uint32_t C_ROW = 32;              // code bytes fetched per W row and stage
constexpr uint32_t C_STAGE = BN * C_ROW;    // 8 KB
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s

struct Smem {
    uint8_t a[STAGES][2][A_SUB];     // X subtiles, 1024-byte aligned
    uint8_t b[STAGES][B_STAGE];      // decoded W tiles
    uint8_t c[STAGES][C_STAGE];      // packed code bytes of the stage (TMA mode)
    uint2 lut[256];                  // byte -> PRMT selectors of its five weights
    uint64_t full_a[STAGES], full_c[STAGES], full_b[STAGES], empty[STAGES], done;
    uint32_t tmem_base;
    int abort_flag;
};

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
// Bounded wait: false when the deadline passed or another role gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kTimeoutNs) {
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

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// PRMT selector byte of one weight: two nibbles naming the bytes of its bf16
// value inside the 8-byte pair (V = {+s, -s}, Z = {0, NaN}).
constexpr uint32_t kSelPos = 0x10, kSelNeg = 0x32, kSelZero = 0x54, kSelNaN = 0x76;

// Decode one row's 64 weights of a stage (columns c0..c0+63 of group g, c0 % 5 == R0)
// into the swizzled tile row.  bytes[] holds code bytes q_lo .. q_lo+13.
template <int R0>
__device__ __forceinline__ void decode_row(const uint2* lut, const uint32_t (&bytes)[14], uint32_t V, uint32_t Z,
                                           uint8_t* tile_row, int row_in_atom) {
    // selector bytes of the 64 columns: column j uses digit (R0 + j) % 5 of byte (R0 + j) / 5
    uint2 e[14];
#pragma unroll
    for (int t = 0; t < 14; ++t) e[t] = lut[bytes[t]];
#pragma unroll
    for (int chunk = 0; chunk < 8; ++chunk) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int j0 = chunk * 8 + 2 * h, j1 = j0 + 1;
            const int q0 = (R0 + j0) / 5, i0 = (R0 + j0) % 5;
            const int q1 = (R0 + j1) / 5, i1 = (R0 + j1) % 5;
            // selector bytes live in byte i of the 8-byte entry {lo, hi}
            uint32_t sel;
            if (q0 == q1) {
                const uint32_t lo = e[q0].x, hi = e[q0].y;
                sel = prmt(lo, hi, (uint32_t)i0 | ((uint32_t)i1 << 4));
            } else {  // pair straddles two bytes: digit 4 of one, digit 0 of the next
                sel = prmt(e[q0].y, e[q1].x, 0u | (4u << 4));
            }
            // sel bytes: [s0, s1, ...]; value selector = s0 | s1 << 8 (PRMT uses the low 16 bits)
            w[h] = prmt(V, Z, sel);
        }
        const int phys = chunk ^ row_in_atom;  // 128-byte swizzle: 16-byte chunk index XOR (row % 8)
        *reinterpret_cast<uint4*>(tile_row + phys * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

struct Params {
    const uint8_t* codes;
    const uint16_t* scales;
    void* Y;
    uint32_t* d_err;
    int64_t M, N;
    int K, G, B, ng;
    int64_t row_bytes;
    int n_tiles;
    int y_bf16;
    int y_vec;  // Y rows allow 16-byte vector stores (base aligned, N a multiple of 16 bytes)
};

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

template <bool CODES_TMA>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                              const __grid_constant__ CUtensorMap tmap_c,
                                                              const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw + ((1024 - (s32(smem_raw) & 1023)) & 1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tile = blockIdx.x / p.n_tiles, n_tile = blockIdx.x % p.n_tiles;
    const int64_t m0 = (int64_t)m_tile * BM, n0 = (int64_t)n_tile * BN;
    const int nk = p.K / BK;
    volatile int* abort_flag = &sm.abort_flag;

    // selector table: byte -> selector bytes of digits 0..4 (bytes 5..7 unused)
    for (int b = threadIdx.x; b < 256; b += kThreads) {
        uint32_t sv[5];
        if (b >= 243) {
            for (int i = 0; i < 5; ++i) sv[i] = kSelNaN;
        } else {
            uint32_t v = b;
            for (int i = 0; i < 5; ++i) {
                const uint32_t d = v % 3;
                v /= 3;
                sv[i] = d == 0 ? kSelNeg : (d == 1 ? kSelZero : kSelPos);
            }
        }
        sm.lut[b] = make_uint2(sv[0] | (sv[1] << 8) | (sv[2] << 16) | (sv[3] << 24), sv[4]);
    }
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
        q_lo = c0 / 5;
    };

    if (warp == 0) {
        // ---------------- TMA producer: X subtiles (and the stage's code window)
        int issued = 0;
        if (lane == 0) {
            for (int kb = 0; kb < nk; ++kb) {
                const int st = kb % STAGES, use = kb / STAGES;
                if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(&sm.full_a[st], 2 * A_SUB);
                tma_load_2d(sm.a[st][0], &tmap_x, kb * BK, (int)m0, &sm.full_a[st]);
                tma_load_2d(sm.a[st][1], &tmap_x, kb * BK, (int)(m0 + UM), &sm.full_a[st]);
                if (CODES_TMA) {
                    int g, c0, q_lo;
                    stage_geom(kb, g, c0, q_lo);
                    const int gb = g * p.B + q_lo;
                    mbar_arrive_expect_tx(&sm.full_c[st], C_STAGE);
                    tma_load_2d(sm.c[st], &tmap_c, gb & ~15, (int)n0, &sm.full_c[st]);
                }
                ++issued;
            }
            // Drain: every issued load must land before the CTA can exit.
            for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb) {
                const int st = kb % STAGES, use = kb / STAGES;
                const uint64_t t0 = globaltimer();
                while (!mbar_try_wait(&sm.full_a[st], use & 1) && globaltimer() - t0 < kTimeoutNs) {
                }
                if (CODES_TMA)
                    while (!mbar_try_wait(&sm.full_c[st], use & 1) && globaltimer() - t0 < kTimeoutNs) {
                    }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: two 128 x 256 x 16 MMAs per k-step
        if (lane == 0) {
            const uint32_t idesc = instr_desc(UM, BN);
            for (int kb = 0; kb < nk; ++kb) {
                const int st = kb % STAGES, use = kb / STAGES;
                if (!mbar_wait(&sm.full_a[st], use & 1, abort_flag)) break;
                if (!mbar_wait(&sm.full_b[st], use & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t b0 = s32(sm.b[st]);
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    const uint32_t a0 = s32(sm.a[st][sub]);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        mma_bf16(tmem + (uint32_t)(sub * BN), smem_desc_sw128(a0 + 32 * k),
                                 smem_desc_sw128(b0 + 32 * k), idesc, (kb > 0 || k > 0) ? 1u : 0u);
                }
                mma_commit(&sm.empty[st]);  // stage free once these MMAs have read it
            }
            mma_commit(&sm.done);  // all issued MMAs complete -> accumulators ready
        }
    } else if (warp >= kDecodeWarp0) {
        // ---------------- decoders: thread -> one W row of the tile
        const int t = threadIdx.x - kDecodeWarp0 * 32;  // 0..255
        const int64_t n = n0 + t;
        const bool row_ok = n < p.N;
        const uint8_t* crow = p.codes + (row_ok ? n : 0) * p.row_bytes;
        const uint16_t* srow = p.scales + (row_ok ? n : 0) * p.ng;
        const int real = p.G - 5 * (p.B - 1);
        const uint32_t pm = padding_mask(real), po = padding_ones(real);
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % STAGES, use = kb / STAGES;
            int g, c0, q_lo;
            stage_geom(kb, g, c0, q_lo);
            uint32_t bytes[14];
            if (CODES_TMA) {
                if (!mbar_wait(&sm.full_c[st], use & 1, abort_flag)) break;
                const int gb = g * p.B + q_lo;
                window_bytes(sm.c[st] + t * C_ROW, gb & 15, bytes);
#pragma unroll
                for (int i = 0; i < 14; ++i)
                    if (q_lo + i >= p.B) bytes[i] = kZeroByte;
            } else {
                if (use > 0 && !mbar_wait(&sm.empty[st], (use - 1) & 1, abort_flag)) break;
                const uint8_t* cb = crow + (int64_t)g * p.B;
#pragma unroll
                for (int i = 0; i < 14; ++i)
                    bytes[i] = (q_lo + i < p.B) ? (uint32_t)__ldg(cb + q_lo + i) : kZeroByte;
            }
            // a group's last byte with a padding digit other than 1 decodes to NaN
            const int ql = p.B - 1 - q_lo;
#pragma unroll
            for (int i = 0; i < 14; ++i) {
                if (i == ql) {
                    const uint32_t dp = byte_digit_pattern(bytes[i]);
                    if ((dp & 0x8000u) == 0 && (dp & pm) != po) bytes[i] = 255;
                }
            }
            const uint32_t sv = __ldg(srow + g);
            uint32_t V, Z;
            if (scale_is_bad(sv)) {
                V = 0x7FC07FC0u;
                Z = 0x7FC07FC0u;
            } else {
                const uint32_t mag = sv == 0 ? 0u : scale_to_bf16_bits((uint16_t)sv);
                V = mag | ((mag ? (mag | 0x8000u) : 0u) << 16);  // {+s, -s}
                Z = 0x7FC00000u;                                // {0, NaN}
            }
            uint8_t* row = sm.b[st] + t * 128;
            const int rin = t & 7;
            switch (c0 % 5) {
                case 0: decode_row<0>(sm.lut, bytes, V, Z, row, rin); break;
                case 1: decode_row<1>(sm.lut, bytes, V, Z, row, rin); break;
                case 2: decode_row<2>(sm.lut, bytes, V, Z, row, rin); break;
                case 3: decode_row<3>(sm.lut, bytes, V, Z, row, rin); break;
                default: decode_row<4>(sm.lut, bytes, V, Z, row, rin); break;
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.full_b[st]);
        }
        // ---------------- epilogue: warps 4..7 read their accumulator quadrant
        if (warp < kDecodeWarp0 + 4) {
            const int q = warp - kDecodeWarp0;  // TMEM lanes 32q .. 32q+31
            const bool ok = mbar_wait(&sm.done, 0, abort_flag);
            tc_fence_after();
            if (ok) {
                for (int sub = 0; sub < 2; ++sub) {
                    const int64_t m = m0 + sub * UM + 32 * q + lane;
                    for (int c = 0; c < BN / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(sub * BN + 32 * c), r);
                        const int64_t nb = n0 + 32 * c;
                        if (m < p.M && nb < p.N) {
                            const int cnt = (int)(p.N - nb < 32 ? p.N - nb : 32);
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
        }
    }

    // ---------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1 && lane == 0 && *abort_flag) {
        // The commit after the issue loop tracks every MMA this CTA issued:
        // wait for it (bounded) before tensor memory is freed.
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&sm.done, 0) && globaltimer() - t0 < kTimeoutNs) {
        }
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 2)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    if (threadIdx.x == 0 && *abort_flag && p.d_err) atomicOr(p.d_err, TQ_DERR_TIMEOUT);
}

// ------------------------------------------------------------------ host

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

size_t gemm_smem_bytes() { return sizeof(gemm::Smem) + 1024; }

cudaError_t launch_gemm_tc(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales, int64_t N,
                           int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err, cudaStream_t stream,
                           int sm_count, bool* handled) {
    using namespace gemm;
    (void)sm_count;
    *handled = false;
    // Shapes this kernel covers: K a multiple of the 64-column stage, G a
    // multiple of 64 (a stage never crosses a group).
    if (K % BK != 0 || G % 64 != 0 || M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (1 << 30))
        return cudaSuccess;
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const int B = bytes_per_group(G);
    const int64_t row_bytes = (int64_t)(K / G) * B;
    CUtensorMap tmap_x, tmap_c;
    std::memset(&tmap_x, 0, sizeof(tmap_x));
    std::memset(&tmap_c, 0, sizeof(tmap_c));
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {BK, UM};
        const cuuint32_t estride[2] = {1, 1};
        CUresult r = enc(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), gdim, gstride, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    // Codes by TMA when their rows are 16-byte multiples and the base is 16-byte aligned.
    const bool codes_tma = (row_bytes % 16 == 0) && ((reinterpret_cast<uintptr_t>(codes) & 15) == 0);
    if (codes_tma) {
        const cuuint64_t gdim[2] = {(cuuint64_t)row_bytes, (cuuint64_t)N};
        const cuuint64_t gstride[1] = {(cuuint64_t)row_bytes};
        const cuuint32_t box[2] = {C_ROW, BN};
        const cuuint32_t estride[2] = {1, 1};
        CUresult r = enc(&tmap_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), gdim, gstride, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    Params p{};
    p.codes = codes;
    p.scales = scales;
    p.Y = Y;
    p.d_err = d_err;
    p.M = M;
    p.N = N;
    p.K = (int)K;
    p.G = G;
    p.B = B;
    p.ng = (int)(K / G);
    p.row_bytes = row_bytes;
    p.n_tiles = (int)((N + BN - 1) / BN);
    p.y_bf16 = y_bf16;
    p.y_vec = ((reinterpret_cast<uintptr_t>(Y) & 15) == 0) && ((N * (y_bf16 ? 2 : 4)) % 16 == 0);
    const int64_t m_tiles = (M + BM - 1) / BM;
    const int64_t grid = m_tiles * p.n_tiles;
    if (grid > 0x7FFFFFFF) return cudaSuccess;
    const size_t smem = gemm_smem_bytes();
    auto kern = codes_tma ? gemm_tc_kernel<true> : gemm_tc_kernel<false>;
    static std::atomic<int> smem_set[2];
    std::atomic<int>& slot = smem_set[codes_tma ? 1 : 0];
    if ((int)smem > slot.load()) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        slot.store((int)smem);
    }
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(tmap_x, tmap_c, p);
    *handled = true;
    return cudaGetLastError();
}

}  // namespace tq
