// gemv_lut_stream.cu -- one-token decode GEMV over large matrices at HBM rate
// (CUDA cores, sm_100a).
//
// Computes Y[n] = sum_g RNE_bf16(s[n,g]) * sum_{j in g} t[n,j] X[j] (tiny-llm
// "Week 2 Day 3: Quantize the Model", "Mathematical Formulation", bias 0, the
// group scale applied once per group as in "Stage 2: SIMD Matvec") for the
// base-3 codes of "precisit/pack-unpack-run" (codec.py: five digits per byte,
// each group byte-aligned) with G = 64 or 128, M = 1, fp32 accumulation.
//
// Lookup tables.  A code byte b covers five activations x_0..x_4 of its group;
// the table of its chunk holds the 243 sums sum_i (d_i(b) - 1) x_i (NaN for
// the 13 invalid byte values and for padding digits other than 1), so one
// byte costs a table load and an add.  512 columns are 104 code bytes at both
// group sizes; a CTA keeps the tables of one such K slice, and the K slices
// of a row are spread over the CTAs of a thread-block cluster whose partial
// rows are added in rank order.
//
// Table layout.  Entry b of a table sits at byte 256 b + 4 slot of its block
// (64 slots of fp32 per entry row, 64 KB per block, two blocks at offset
// 0x10000 of the CTA's shared-memory window), so slot s lives in bank s mod 32
// whatever b is.  A PRMT builds the whole lookup address in one instruction:
// it places the code byte in bits 8..15, the lane's slot offset (4 x bank,
// +128 for the upper 32 slots) in bits 0..7, the block in bits 16..23 and the
// window's base in bits 24..31 (in a cluster, a CTA's shared-memory window
// starts at rank x 2^24: the address of rank 1's first dynamic byte is
// 0x1000400), all from one per-lane constant register.
//
// Lanes.  Each lane reads one code word of a row's K slice with a single
// global load and owns the bytes of ONE group in it, so one scale per lane
// and row suffices: words that straddle a group boundary are read by two
// lanes, each of which masks the other group's bytes by pointing their
// lookups at an all-zero table column.
//   G = 128: 8-byte words, 13 words + 3 straddling copies = 16 lanes per
//            row, two rows per warp step; the second row's lanes take their
//            bytes in the order 4..7, 0..3 so that the 32 lookups of an
//            instruction hit 32 different banks.
//   G = 64:  4-byte words, 26 words + 6 straddling copies = 32 lanes, one
//            row per warp step.
// A warp handles 32 rows per chunk (16 or 32 steps) and keeps the code words
// of U steps in flight (ld.global.nc, no L1 allocation); the row stride is a
// compile-time constant (one kernel per cluster size), so the loads of a
// chunk walk one pointer with immediate offsets.  Two steps are summed side
// by side in packed fp32 pairs (add.rn.f32x2), in the same order as one step
// alone.  A warp's per-row partials are summed across lanes by a transposing
// butterfly; steps past the warp's last row compute rows that are never
// stored, so no step is predicated.
//
// K slices.  Row j of a cluster round belongs to rank j mod CS; each warp
// stores the partial of its slice straight into the owner's shared memory
// (st.shared::cluster), and after one cluster barrier per round the owner
// adds the CS partials in rank order and writes Y.
//
// Other formats.  The same kernel reads 2-bit codes (a byte is four codes,
// 81 valid entries, NaN for any code 3) and the affine 4-bit codes of the
// W4A16 format (tiny-llm "Week 2 Day 3: Quantize the Model", "Group-Wise
// Affine Quantization"): a byte is two codes q0 (low nibble) and q1, its
// entry q0 x_0 + q1 x_1 over all 256 values, so a CTA's 128 table slots cover
// 256 columns; a lane's step is s S + b Xw, S its table sum, s and b the
// group's bf16 scale and bias and Xw the sum of the lane's 16 activations, so
// the lanes of a group add up to s sum q x + b sum x.
//
// Ordering.  Codes and scales do not depend on earlier kernels: the first
// steps' loads and the constant parts of the tables (the masking columns,
// the invalid-byte rows) are issued before griddepcontrol.wait; the
// activations, and therefore the table values, only after it.  A NaN output
// row (invalid byte, bad padding, bad scale) is rescanned for its error bits.
#include <cooperative_groups.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "tq_internal.cuh"

namespace cg = cooperative_groups;

namespace tq {

namespace {

constexpr int kLsThreads = 512;
constexpr int kLsWarps = kLsThreads / 32;
constexpr uint32_t kLsTableAbs = 0x10000u;   // offset of the tables in the CTA's shared-memory window
constexpr uint32_t kLsBlockBytes = 0x10000u; // one block: 256 entry rows x 64 slots x 4 B
constexpr uint32_t kLsSmemBytes = 0x30000u;  // dynamic request: covers [base, 0x30000) for any base <= 0x10000
constexpr int kLsSliceCols = 512;            // K columns per CTA
constexpr int kLsRound = 4096;               // rows per cluster round (partials in shared memory)
constexpr int kLsFreeBank = 26;              // banks 26..31: all-zero columns for masked lookups
constexpr int kLsChunkRows = 32;             // rows per warp chunk
constexpr int kLsScaleStride = 36;           // floats per group in a warp's scale block
static_assert(kLsThreads == kLsSliceCols, "at most one activation of the slice per thread");

// FMT 3: base-3 codes (five digits per byte, 104 bytes per 512 columns);
// FMT 2: 2-bit codes (four per byte, 128 bytes per 512 columns, groups of
// 64 or 128 columns are whole 8-byte words); FMT 4: the affine 4-bit codes
// (two per byte, 128 bytes per 256 columns, groups whole 8-byte words).
template <int G, int FMT>
struct LsCfg;
template <>
struct LsCfg<128, 3> {
    static constexpr int B = 26;    // code bytes per group
    static constexpr int SB = 104;  // code bytes per slice
    static constexpr int GPS = 4;   // groups per slice
    static constexpr int RPS = 2;   // rows per warp step
    static constexpr int SPC = 16;  // steps per chunk
    static constexpr int U = 8;     // steps of code loads in flight
};
template <>
struct LsCfg<64, 3> {
    static constexpr int B = 13, SB = 104, GPS = 8, RPS = 1, SPC = 32, U = 8;
};
template <>
struct LsCfg<128, 2> {
    static constexpr int B = 32, SB = 128, GPS = 4, RPS = 2, SPC = 16, U = 8;
};
template <>
struct LsCfg<64, 2> {
    static constexpr int B = 16, SB = 128, GPS = 8, RPS = 2, SPC = 16, U = 8;
};
template <>
struct LsCfg<128, 4> {
    static constexpr int B = 64, SB = 128, GPS = 2, RPS = 2, SPC = 16, U = 8;
};
template <>
struct LsCfg<64, 4> {
    static constexpr int B = 32, SB = 128, GPS = 4, RPS = 2, SPC = 16, U = 8;
};
// K columns of one CTA's tables: 128 table slots, one per code byte
template <int FMT>
__host__ __device__ constexpr int ls_slice_cols() { return FMT == 4 ? 256 : kLsSliceCols; }
// 8-byte code words, two rows per step
template <int G, int FMT>
constexpr bool ls_wide() { return LsCfg<G, FMT>::RPS == 2; }

// Shared memory below the tables: per-warp decoded scales of a chunk (stored
// group-major, and within a group in step order for each row of the step,
// kLsScaleStride floats per group so that the float4 reads of lanes of
// different groups and rows land in different banks; FMT 4 adds the biases
// in a second such block), then two buffers of
// partial rows (CS slots of kLsRound / CS rows each, alternating by round),
// then the slice's activations in fp32.
constexpr int kLsPartFloats = kLsRound + 8;
template <int G, int FMT>
__host__ __device__ constexpr uint32_t ls_scale_bytes() {
    return (uint32_t)kLsWarps * LsCfg<G, FMT>::GPS * kLsScaleStride * 4 * (FMT == 4 ? 2 : 1);
}
template <int G, int FMT>
__host__ __device__ constexpr uint32_t ls_misc_bytes() {
    return ls_scale_bytes<G, FMT>() + 2u * kLsPartFloats * 4 + (uint32_t)(kLsSliceCols + kLsSliceCols / 32) * 4;
}

// Index of activation c of the slice in the staged copy: one padding float
// after every 32, so that the build's lanes, which read columns 20 or 32
// apart, spread over the banks.
__device__ __forceinline__ int xs_at(int c) { return c + (c >> 5); }

struct LsArgs {
    const uint16_t* X;
    const uint8_t* codes;
    const uint16_t* scales;
    const uint16_t* biases;  // FMT 4 only
    int64_t N;
    int K, CS;
    int64_t rows_per_cluster;
    void* Y;
    int y_bf16;
    uint32_t* d_err;
};

// Table slot of chunk position p of a slice (p < 104 base-3, < 128 2-bit), as
// the lanes below read it: 8-byte words: p = 8 w + j -> block (j & 3) >> 1,
// upper slots j & 1, bank 2 w + (j >> 2); 4-byte words (base-3, G = 64):
// p = 4 w + j -> block j >> 1, upper slots j & 1, bank w.  The table build
// needs the inverse: the position held at (block, sub, bank).
template <int G, int FMT>
__device__ __forceinline__ int ls_slot_position(int block, int sub, int bank) {
    if constexpr (ls_wide<G, FMT>()) return 8 * (bank >> 1) + 4 * (bank & 1) + 2 * block + sub;
    else return 4 * bank + 2 * block + sub;
}

// Per-lane constants: offset of the lane's word in the slice, the row within
// the step, the lane's group in the slice and the PRMT source words of its
// lookups: lb[i] = {slot offset of lookup 2i (4 x bank), of lookup 2i + 1
// (128 + 4 x bank: the upper slots), table block of both (bits 16..23 of the
// address), window base >> 24}.
struct LsLane {
    uint32_t wofs;
    int h, grp;
    uint32_t lb[4];
};

template <int G, int FMT>
__device__ __forceinline__ LsLane ls_lane(int lane, uint32_t win_base) {
    LsLane L{};
    for (int i = 0; i < 4; ++i) {
        const uint32_t block = ls_wide<G, FMT>() ? (uint32_t)(i & 1) : (uint32_t)i;  // lookups 2i, 2i + 1
        L.lb[i] = (win_base & 0xFF000000u) | (((kLsTableAbs + block * kLsBlockBytes) >> 16) << 16) | 0x8000u;
    }
    if constexpr (FMT == 2 || FMT == 4) {
        // 16 words per row, no group straddles a word: every lookup is live
        const int h = lane >> 4, w = lane & 15;
        for (int k = 0; k < 8; ++k) {
            const int j = h ? ((k + 4) & 7) : k;
            L.lb[k >> 1] |= (uint32_t)(4 * (2 * w + (j >> 2))) << (8 * (k & 1));
        }
        L.wofs = 8u * w;
        L.h = h;
        L.grp = 8 * w / LsCfg<G, FMT>::B;
    } else if constexpr (G == 128) {
        const int h = lane >> 4, q = lane & 15;
        const int w = q < 13 ? q : 3 * (q - 12);  // copies of the straddling words 3, 6, 9
        const bool copy = q >= 13;
        const int si = (w == 3 || w == 6 || w == 9) ? w / 3 - 1 : 0;
        const int grp = copy ? (8 * w + 7) / 26 : (8 * w) / 26;
        for (int k = 0; k < 8; ++k) {
            const int j = h ? ((k + 4) & 7) : k;
            const bool live = (8 * w + j) / 26 == grp;
            const int bank = live ? 2 * w + (j >> 2) : kLsFreeBank + 2 * si + h;
            L.lb[k >> 1] |= (uint32_t)(4 * bank) << (8 * (k & 1));
        }
        L.wofs = 8u * w;
        L.h = h;
        L.grp = grp;
    } else {
        // straddling words 3, 6, 9, 16, 19, 22 (copy i = lane - 26)
        const bool copy = lane >= 26;
        const int w = copy ? (lane < 29 ? 3 * (lane - 25) : 3 * (lane - 26) + 7) : lane;
        const int si = w <= 9 ? w / 3 - 1 : (w - 7) / 3;
        const int grp = copy ? (4 * w + 3) / 13 : (4 * w) / 13;
        for (int k = 0; k < 4; ++k) {
            const bool live = (4 * w + k) / 13 == grp;
            const int bank = live ? w : kLsFreeBank + si;
            L.lb[k >> 1] |= (uint32_t)(4 * bank) << (8 * (k & 1));
        }
        L.wofs = 4u * w;
        L.h = 0;
        L.grp = grp;
    }
    return L;
}

__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
template <uint32_t IMM>
__device__ __forceinline__ float lds_imm(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(IMM));
    return v;
}
__device__ __forceinline__ uint2 ldg_nc_u2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// One lookup: the whole shared-memory address from one PRMT -- byte K mod 4
// of word `a` as bits 8..15, the slot byte K mod 2 of `lb` as bits 0..7 and
// bytes 2, 3 of `lb` (table block, window base) above.
template <int K>
__device__ __forceinline__ float ls_lookup(uint32_t a, uint32_t lb) {
    constexpr uint32_t kk = (uint32_t)(K & 3);
    constexpr uint32_t sel = 0x7600u | (kk << 4) | (4u + (uint32_t)(K & 1));
    return lds_imm<0>(prmt32(a, lb, sel));
}

// Decoded scale as the matmul uses it: fp32 of RNE_bf16(binary16 s); NaN for
// a rejected scale (sign bit set, Inf or NaN: every pattern >= 0x7C00).
__device__ __forceinline__ float ls_scale(uint32_t s) {
    const float r = __bfloat162float(__float2bfloat16_rn(__half2float(__ushort_as_half((unsigned short)s))));
    return s >= 0x7C00u ? __uint_as_float(0x7FC00000u) : r;
}

// Transposing butterfly within aligned groups of NV lanes (NV = 16 or 32):
// on exit lane l holds the sum over its group of v[l mod NV].  The adds of a
// level run in packed pairs; each is the same single fp32 add as unpacked.
template <int NV>
__device__ __forceinline__ float ls_transpose_reduce(float (&v)[NV], int lane) {
#pragma unroll
    for (int n = NV / 2; n >= 1; n >>= 1) {
        const bool upper = (lane & n) != 0;
        float keep[NV / 2], recv[NV / 2];
#pragma unroll
        for (int i = 0; i < n; ++i) {
            keep[i] = upper ? v[n + i] : v[i];
            recv[i] = __shfl_xor_sync(0xffffffffu, upper ? v[i] : v[n + i], n);
        }
        if (n >= 2) {
#pragma unroll
            for (int i = 0; i < n; i += 2) {
                const float2 r = f2_unpack(f2_add(f2_pack(keep[i], keep[i + 1]), f2_pack(recv[i], recv[i + 1])));
                v[i] = r.x;
                v[i + 1] = r.y;
            }
        } else {
            v[0] = keep[0] + recv[0];
        }
    }
    return v[0];
}

// Code word of one lane and step.
template <bool WIDE>
using LsWord = typename std::conditional<WIDE, uint2, uint32_t>::type;
template <bool WIDE>
__device__ __forceinline__ LsWord<WIDE> ls_load(const uint8_t* p) {
    if constexpr (WIDE) return ldg_nc_u2(p);
    else return ldg_nc_u32(p);
}

// The table sums of two steps' code words (wa, wb), side by side (packed):
// ((t0+t1)+(t2+t3)) + ((t4+t5)+(t6+t7)) per step.
template <bool WIDE>
__device__ __forceinline__ uint64_t ls_two_sums(const LsWord<WIDE>& wa, const LsWord<WIDE>& wb, const LsLane& L) {
    if constexpr (WIDE) {
        const uint32_t a0 = L.h ? wa.y : wa.x, a1 = L.h ? wa.x : wa.y;
        const uint32_t b0 = L.h ? wb.y : wb.x, b1 = L.h ? wb.x : wb.y;
        const uint64_t p0 = f2_pack(ls_lookup<0>(a0, L.lb[0]), ls_lookup<0>(b0, L.lb[0]));
        const uint64_t p1 = f2_pack(ls_lookup<1>(a0, L.lb[0]), ls_lookup<1>(b0, L.lb[0]));
        const uint64_t p2 = f2_pack(ls_lookup<2>(a0, L.lb[1]), ls_lookup<2>(b0, L.lb[1]));
        const uint64_t p3 = f2_pack(ls_lookup<3>(a0, L.lb[1]), ls_lookup<3>(b0, L.lb[1]));
        const uint64_t p4 = f2_pack(ls_lookup<4>(a1, L.lb[2]), ls_lookup<4>(b1, L.lb[2]));
        const uint64_t p5 = f2_pack(ls_lookup<5>(a1, L.lb[2]), ls_lookup<5>(b1, L.lb[2]));
        const uint64_t p6 = f2_pack(ls_lookup<6>(a1, L.lb[3]), ls_lookup<6>(b1, L.lb[3]));
        const uint64_t p7 = f2_pack(ls_lookup<7>(a1, L.lb[3]), ls_lookup<7>(b1, L.lb[3]));
        const uint64_t lo = f2_add(f2_add(p0, p1), f2_add(p2, p3));
        const uint64_t hi = f2_add(f2_add(p4, p5), f2_add(p6, p7));
        return f2_add(lo, hi);
    } else {
        const uint64_t p0 = f2_pack(ls_lookup<0>(wa, L.lb[0]), ls_lookup<0>(wb, L.lb[0]));
        const uint64_t p1 = f2_pack(ls_lookup<1>(wa, L.lb[0]), ls_lookup<1>(wb, L.lb[0]));
        const uint64_t p2 = f2_pack(ls_lookup<2>(wa, L.lb[1]), ls_lookup<2>(wb, L.lb[1]));
        const uint64_t p3 = f2_pack(ls_lookup<3>(wa, L.lb[1]), ls_lookup<3>(wb, L.lb[1]));
        return f2_add(f2_add(p0, p1), f2_add(p2, p3));
    }
}

// Packed raw scales of one row's groups in a slice (2 bytes per group).
template <int BYTES>
using LsRaw = typename std::conditional<BYTES == 4, uint32_t,
                                        typename std::conditional<BYTES == 8, uint2, uint4>::type>::type;

__device__ __forceinline__ void st_cluster_f32(uint32_t local_addr, int rank, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

template <int G, int FMT, int CS>
__global__ void __launch_bounds__(kLsThreads, 1) gemv_lut_stream_kernel(const LsArgs a) {
    using C = LsCfg<G, FMT>;
    constexpr bool WIDE = ls_wide<G, FMT>();
    using Word = LsWord<WIDE>;
    constexpr int SPC = C::SPC, U = C::U, RPS = C::RPS, GPS = C::GPS;
    constexpr int64_t RB = (int64_t)CS * C::SB;          // code bytes per row
    constexpr int NG = CS * GPS;                         // groups per row
    constexpr int64_t STEP = RPS * RB;                   // code bytes between a lane's consecutive steps
    constexpr int PS = (kLsRound + CS - 1) / CS;         // partial rows per rank slot
    static_assert(U % 2 == 0 && SPC % U == 0, "steps run in pairs; the load ring divides a chunk");
    static_assert(CS * PS <= kLsPartFloats, "partial buffer");
    extern __shared__ __align__(16) unsigned char smem[];
    const int crank = (int)cg::this_cluster().block_rank();
    const int cid = (int)(blockIdx.x / (unsigned)CS);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // Shared-memory window (base: the top byte of the dynamic region's
    // address, the CTA's rank in the cluster): the tables at offsets
    // [0x10000, 0x30000), the scales, partials and activations just below.
    const uint32_t dyn = (uint32_t)__cvta_generic_to_shared(smem);
    const uint32_t wbase = dyn & 0xFF000000u, doff = dyn - wbase;
    const uint32_t misc = kLsTableAbs - ls_misc_bytes<G, FMT>();
    if (doff > misc) {  // the same offset in every CTA: all of them leave here, none waits on a peer
        if (threadIdx.x == 0 && a.d_err) atomicOr(a.d_err, TQ_DERR_TIMEOUT);
        return;
    }
    // peers store partial rows into this CTA only after the matching wait
    cluster_arrive_relaxed();
    float* ssc = reinterpret_cast<float*>(smem + (misc - doff)) + warp * GPS * kLsScaleStride * (FMT == 4 ? 2 : 1);
    float* part = reinterpret_cast<float*>(smem + (misc - doff) + ls_scale_bytes<G, FMT>());
    float* xs = part + 2 * kLsPartFloats;
    const uint32_t part_sa = (uint32_t)__cvta_generic_to_shared(part);
    const uint32_t tabs = wbase + kLsTableAbs;  // the tables, for the stores of the build
    const float nan = __uint_as_float(0x7FC00000u);

    if constexpr (FMT == 3) {
        // constant parts of the tables: the masking columns (banks 26..31) and
        // the invalid-byte rows 243..255 (NaN in the table columns)
        for (int it = warp; it < 36; it += kLsWarps) {
            if (lane >= kLsFreeBank) {
                const int bs = it / 9, d34 = it - 9 * bs;
                const uint32_t base =
                    tabs + (bs >> 1) * kLsBlockBytes + 27u * d34 * 256u + 4u * (uint32_t)(lane + 32 * (bs & 1));
#pragma unroll
                for (int e = 0; e < 27; ++e) sts_f32(base + 256u * e, 0.f);
            }
        }
        for (int it = warp; it < 4; it += kLsWarps) {
            const uint32_t base = tabs + (it >> 1) * kLsBlockBytes + 4u * (uint32_t)(lane + 32 * (it & 1));
            const float v = lane < kLsFreeBank ? nan : 0.f;
#pragma unroll
            for (int b = 243; b < 256; ++b) sts_f32(base + 256u * b, v);
        }
    } else if constexpr (FMT == 2) {
        // constant parts of the tables: every byte with a code 3 is invalid (NaN);
        // warp item (block, sub, c2, c3): entries b = c0 + 4 c1 + 16 c2 + 64 c3
        for (int it = warp; it < 64; it += kLsWarps) {
            const int bs = it >> 4, c2 = it & 3, c3 = (it >> 2) & 3;
            const uint32_t base = tabs + (bs >> 1) * kLsBlockBytes + 4u * (uint32_t)(lane + 32 * (bs & 1)) +
                                  256u * (uint32_t)(16 * c2 + 64 * c3);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (c2 == 3 || c3 == 3 || (e & 3) == 3 || (e >> 2) == 3) sts_f32(base + 256u * e, nan);
        }
    }

    const LsLane L = ls_lane<G, FMT>(lane, wbase);
    const int64_t crow0 = (int64_t)cid * a.rows_per_cluster;
    const int64_t crow1 = min(a.N, crow0 + a.rows_per_cluster);
    const uint8_t* cbase = a.codes + (int64_t)crank * C::SB + L.wofs;
    const uint16_t* sbase = a.scales + (int64_t)crank * GPS;
    const uint16_t* bbase = a.biases + (int64_t)crank * GPS;  // FMT 4
    // this lane's scales in the warp's block: group L.grp, row L.h of each step, steps in order
    const float4* ssc_lane = reinterpret_cast<const float4*>(ssc + L.grp * kLsScaleStride + (RPS == 2 ? 16 * L.h : 0));
    constexpr int kBiasF4 = GPS * kLsScaleStride / 4;  // FMT 4: the biases' block, in float4 past the scales'
    float xw = 0.f;  // FMT 4: sum of the activations of the lane's 16 columns
    const int res_row = WIDE ? 2 * (lane & 15) + (lane >> 4) : lane;  // row of the reduced value, in the chunk
    uint32_t err_acc = 0;
    bool tables_built = false;
    int round = 0;

    for (int64_t rr0 = crow0; rr0 < crow1; rr0 += kLsRound, ++round) {
        const int nround = (int)(crow1 - rr0 < (int64_t)kLsRound ? crow1 - rr0 : (int64_t)kLsRound);
        // this warp's rows of the round
        int per = (nround + kLsWarps - 1) / kLsWarps;
        per = (per + RPS - 1) / RPS * RPS;
        const int wlo = min(nround, warp * per), whi = min(nround, wlo + per);
        const int nr = whi - wlo;
        const int64_t wr0 = rr0 + wlo;
        const int T = (nr + RPS - 1) / RPS;
        const int nch = (T + SPC - 1) / SPC;
        const uint32_t pbuf = part_sa + (uint32_t)(round & 1) * kLsPartFloats * 4u;

        // code word of step t, the row clamped to the warp's last
        auto load_clamped = [&](int t) -> Word {
            int r = RPS * t + L.h;
            r = r < nr ? r : nr - 1;
            return ls_load<WIDE>(cbase + (wr0 + r) * RB);
        };
        using SRaw = LsRaw<2 * GPS>;
        auto load_scales = [&](const uint16_t* base, int ch) -> SRaw {
            int r = ch * kLsChunkRows + lane;
            r = r < nr ? r : nr - 1;
            return __ldg(reinterpret_cast<const SRaw*>(base + (wr0 + r) * NG));
        };

        Word cb[U];
        SRaw sraw{}, braw{};
        if (nr > 0) {
#pragma unroll
            for (int u = 0; u < U; ++u) cb[u] = load_clamped(u);
            sraw = load_scales(sbase, 0);
            if constexpr (FMT == 4) braw = load_scales(bbase, 0);
        }

        if (!tables_built) {
            // Activations come from the preceding kernel: everything above ran
            // before this wait.  One coalesced read of the slice's 512
            // activations (every CTA of the grid reads the same 1 KB, so the
            // per-entry reads of the build go to shared memory).
            asm volatile("griddepcontrol.wait;" ::: "memory");
            constexpr int SC = ls_slice_cols<FMT>();
            if (threadIdx.x < SC)
                xs[xs_at(threadIdx.x)] = __uint_as_float((uint32_t)__ldcg(a.X + crank * SC + threadIdx.x) << 16);
            __syncthreads();
            if constexpr (FMT == 3) {
                // warp item (block, sub, d3 + 3 d4): the 27 entries b = d0 + 3 d1 + 9 d2 + 27 (d3 + 3 d4)
                // of one table row per lane (lane = bank)
                for (int it = warp; it < 36; it += kLsWarps) {
                    if (lane < kLsFreeBank) {
                        const int bs = it / 9, d34 = it - 9 * bs;
                        const int block = bs >> 1, sub = bs & 1;
                        const uint32_t base = tabs + block * kLsBlockBytes + 27u * d34 * 256u +
                                              4u * (uint32_t)(lane + 32 * sub);
                        const int p = ls_slot_position<G, FMT>(block, sub, lane);
                        const int g = p / C::B, j = p - g * C::B;
                        const int real = min(5, G - 5 * j);
                        const int c0 = g * G + 5 * j;
                        float x[5];
#pragma unroll
                        for (int i = 0; i < 5; ++i) x[i] = i < real ? xs[xs_at(c0 + i)] : 0.f;
                        const int d3 = d34 % 3, d4 = d34 / 3;
                        const bool bad34 = (3 >= real && d3 != 1) || (4 >= real && d4 != 1);
                        const float h34 = bad34 ? nan : (float)(d3 - 1) * x[3] + (float)(d4 - 1) * x[4];
                        float P[9];
#pragma unroll
                        for (int d1 = 0; d1 < 3; ++d1)
#pragma unroll
                            for (int d0 = 0; d0 < 3; ++d0) {
                                const bool bad = (1 >= real && d1 != 1) || (0 >= real && d0 != 1);
                                P[d0 + 3 * d1] = bad ? nan : (float)(d0 - 1) * x[0] + (float)(d1 - 1) * x[1];
                            }
#pragma unroll
                        for (int d2 = 0; d2 < 3; ++d2) {
                            const bool bad2 = 2 >= real && d2 != 1;
                            const float q2 = bad2 ? nan : h34 + (float)(d2 - 1) * x[2];
#pragma unroll
                            for (int e = 0; e < 9; ++e) sts_f32(base + 256u * (9 * d2 + e), P[e] + q2);
                        }
                    }
                }
            } else if constexpr (FMT == 4) {
                // warp item (block, sub, q1): the 16 entries b = q0 + 16 q1 of one
                // table row per lane (lane = bank), q0 x[2p] + q1 x[2p + 1]
                for (int it = warp; it < 64; it += kLsWarps) {
                    const int bs = it >> 4, q1 = it & 15;
                    const int block = bs >> 1, sub = bs & 1;
                    const uint32_t base = tabs + block * kLsBlockBytes + 4u * (uint32_t)(lane + 32 * sub) +
                                          256u * (uint32_t)(16 * q1);
                    const int c0 = 2 * ls_slot_position<G, FMT>(block, sub, lane);
                    const float hi = (float)q1 * xs[xs_at(c0 + 1)], x0 = xs[xs_at(c0)];
#pragma unroll
                    for (int q0 = 0; q0 < 16; ++q0) sts_f32(base + 256u * (uint32_t)q0, __fmaf_rn((float)q0, x0, hi));
                }
                // the lane's columns 16 w .. 16 w + 15 of the slice
#pragma unroll
                for (int i = 0; i < 16; ++i) xw += xs[xs_at(2 * (int)L.wofs + i)];
            } else {
                // warp item (block, sub, c2 + 3 c3), c2, c3 < 3: the 9 valid entries
                // b = c0 + 4 c1 + 16 c2 + 64 c3 (c0, c1 < 3) of one table row per lane (lane = bank)
                for (int it = warp; it < 36; it += kLsWarps) {
                    const int bs = it / 9, c23 = it - 9 * bs, c2 = c23 % 3, c3 = c23 / 3;
                    const int block = bs >> 1, sub = bs & 1;
                    const uint32_t base = tabs + block * kLsBlockBytes + 4u * (uint32_t)(lane + 32 * sub) +
                                          256u * (uint32_t)(16 * c2 + 64 * c3);
                    const int c0 = 4 * ls_slot_position<G, FMT>(block, sub, lane);
                    float xp[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) xp[i] = xs[xs_at(c0 + i)];
                    const float q = (float)(c2 - 1) * xp[2] + (float)(c3 - 1) * xp[3];
#pragma unroll
                    for (int c1 = 0; c1 < 3; ++c1)
#pragma unroll
                        for (int c0 = 0; c0 < 3; ++c0)
                            sts_f32(base + 256u * (uint32_t)(c0 + 4 * c1),
                                    ((float)(c0 - 1) * xp[0] + (float)(c1 - 1) * xp[1]) + q);
                }
            }
            __syncthreads();
            cluster_wait();  // every CTA of the cluster runs: partials may be stored into peers
            tables_built = true;
        }

        // Chunk ch of the warp.  WALK: every load the chunk issues (U steps
        // ahead) stays inside the matrix, so the loads walk one pointer with
        // immediate offsets (rows past the warp's own are read and their
        // results never stored); otherwise each load is clamped to the warp's
        // last row.
        const uint8_t* lp = cbase + (wr0 + RPS * U + L.h) * RB;
        auto run_chunk = [&](int ch, auto walk_tag) {
            constexpr bool WALK = decltype(walk_tag)::value;
            // decoded scales of this chunk's 32 rows (lane = row), stored by group
            {
                const uint32_t* sw = reinterpret_cast<const uint32_t*>(&sraw);
                const int col = RPS == 2 ? 16 * (lane & 1) + (lane >> 1) : lane;
#pragma unroll
                for (int g = 0; g < GPS; ++g) {
                    const uint32_t raw = g & 1 ? sw[g >> 1] >> 16 : sw[g >> 1] & 0xFFFFu;
                    // FMT 4: bf16 scale and bias, taken as they are
                    ssc[g * kLsScaleStride + col] = FMT == 4 ? __uint_as_float(raw << 16) : ls_scale(raw);
                }
                if constexpr (FMT == 4) {
                    const uint32_t* bw = reinterpret_cast<const uint32_t*>(&braw);
#pragma unroll
                    for (int g = 0; g < GPS; ++g)
                        ssc[(GPS + g) * kLsScaleStride + col] =
                            __uint_as_float((g & 1 ? bw[g >> 1] >> 16 : bw[g >> 1] & 0xFFFFu) << 16);
                }
                if (ch + 1 < nch) {
                    sraw = load_scales(sbase, ch + 1);
                    if constexpr (FMT == 4) braw = load_scales(bbase, ch + 1);
                }
                __syncwarp();
            }
            float v[SPC];
            float4 sc4;
            [[maybe_unused]] float4 bi4;
#pragma unroll
            for (int s = 0; s < SPC; s += 2) {
                const Word wa = cb[s % U], wb = cb[(s + 1) % U];
                if constexpr (WALK) {
                    cb[s % U] = ls_load<WIDE>(lp + s * STEP);
                    cb[(s + 1) % U] = ls_load<WIDE>(lp + (s + 1) * STEP);
                } else {
                    cb[s % U] = load_clamped(ch * SPC + s + U);
                    cb[(s + 1) % U] = load_clamped(ch * SPC + s + 1 + U);
                }
                if (s % 4 == 0) {
                    sc4 = ssc_lane[s / 4];
                    if constexpr (FMT == 4) bi4 = ssc_lane[kBiasF4 + s / 4];
                }
                const uint64_t sum = ls_two_sums<WIDE>(wa, wb, L);
                const uint64_t sc = s % 4 == 0 ? f2_pack(sc4.x, sc4.y) : f2_pack(sc4.z, sc4.w);
                float2 r;
                if constexpr (FMT == 4) {
                    // s S + b Xw: the lane's share of the group's bias term
                    const uint64_t bi = s % 4 == 0 ? f2_pack(bi4.x, bi4.y) : f2_pack(bi4.z, bi4.w);
                    r = f2_unpack(f2_fma(sum, sc, f2_mul(bi, f2_pack(xw, xw))));
                } else {
                    r = f2_unpack(f2_mul(sum, sc));
                }
                v[s] = r.x;
                v[s + 1] = r.y;
            }
            if constexpr (WALK) lp += SPC * STEP;
            __syncwarp();  // this chunk's scales are consumed before the next chunk rewrites them
            const float tot = ls_transpose_reduce<SPC>(v, lane);
            const int r = ch * kLsChunkRows + res_row;
            if (r < nr) {
                const int j = wlo + r;  // row within the round: owner rank j mod CS, slot j / CS
                st_cluster_f32(pbuf + 4u * (uint32_t)(crank * PS + j / CS), j % CS, tot);
            }
        };
        // chunk ch walks while its last load, row wr0 + RPS ((ch + 1) SPC + U) - 1, is below N
        const int64_t walk_rows = a.N - wr0 - (int64_t)RPS * U;
        int ch = 0;
        for (; ch < nch && (int64_t)RPS * (ch + 1) * SPC <= walk_rows; ++ch) run_chunk(ch, std::true_type{});
        for (; ch < nch; ++ch) run_chunk(ch, std::false_type{});

        // K slices: every rank's partials of the round are stored, then each
        // rank adds the partials of its rows (j = crank mod CS) in rank order.
        cluster_arrive();
        cluster_wait();
        const int own = (nround - crank + CS - 1) / CS;
        const float* pb = reinterpret_cast<const float*>(smem + (misc - doff) + ls_scale_bytes<G, FMT>()) +
                          (round & 1) * kLsPartFloats;
        for (int i = (int)threadIdx.x; i < own; i += kLsThreads) {
            float y = 0.f;
#pragma unroll
            for (int q = 0; q < CS; ++q) y += pb[q * PS + i];
            const int64_t n = rr0 + crank + (int64_t)CS * i;
            if (y != y) {
                if constexpr (FMT == 3) err_acc |= scan_row_errors(a.codes + n * RB, a.scales + n * NG, NG, G, C::B);
                else if constexpr (FMT == 2) err_acc |= scan_row_errors2(a.codes + n * RB, a.scales + n * NG, NG, G);
            }
            if (a.y_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[n] = __float2bfloat16_rn(y);
            else reinterpret_cast<float*>(a.Y)[n] = y;
        }
    }
    if (!tables_built) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        cluster_wait();
    }
    if (err_acc && a.d_err) atomicOr(a.d_err, err_acc);
}

template <int G, int FMT, int CS>
cudaError_t launch_ls(const LsArgs& a0, cudaStream_t stream, int sm_count) {
    auto kern = gemv_lut_stream_kernel<G, FMT, CS>;
    static SmemAttr smem_attr;
    static int max_clusters = 0;
    static std::mutex mu;
    if (cudaError_t e = smem_attr.ensure(kern, (int)kLsSmemBytes)) return e;
    LsArgs a = a0;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kLsThreads);
    cfg.dynamicSmemBytes = kLsSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    int ncl;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (max_clusters == 0) {
            cfg.gridDim = dim3((unsigned)(CS * (sm_count / CS)));
            int n = 0;
            cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
            if (e != cudaSuccess) return e;
            max_clusters = n > 0 ? n : 1;
        }
        ncl = max_clusters;
    }
    const int64_t want = (a.N + 63) / 64;  // at least 64 rows per cluster
    if (want < ncl) ncl = (int)(want < 1 ? 1 : want);
    a.rows_per_cluster = (a.N + ncl - 1) / ncl;
    cfg.gridDim = dim3((unsigned)(ncl * CS));
    static const bool debug = getenv("TQ_DEBUG_PLAN") != nullptr;
    if (debug)
        fprintf(stderr, "tq gemv_lut_stream fmt=%d N=%lld K=%d G=%d: CS=%d clusters=%d rows/cluster=%lld\n", FMT,
                (long long)a.N, a.K, G, CS, ncl, (long long)a.rows_per_cluster);
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int G, int FMT>
cudaError_t launch_ls_cs(const LsArgs& a, cudaStream_t stream, int sm_count) {
    switch (a.CS) {
        case 1: return launch_ls<G, FMT, 1>(a, stream, sm_count);
        case 2: return launch_ls<G, FMT, 2>(a, stream, sm_count);
        case 3: return launch_ls<G, FMT, 3>(a, stream, sm_count);
        case 4: return launch_ls<G, FMT, 4>(a, stream, sm_count);
        case 5: return launch_ls<G, FMT, 5>(a, stream, sm_count);
        case 6: return launch_ls<G, FMT, 6>(a, stream, sm_count);
        case 7: return launch_ls<G, FMT, 7>(a, stream, sm_count);
        case 8: return launch_ls<G, FMT, 8>(a, stream, sm_count);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

// fmt 3: base-3 codes, fmt 2: 2-bit codes.  Returns cudaErrorNotSupported
// when the shape is not covered: M != 1, G not 64 or 128, K not a multiple
// of 512 or above 4096, or unaligned codes/scales.
cudaError_t launch_gemv_lut_stream(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                                   int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                                   cudaStream_t stream, int sm_count, int fmt) {
    if (M != 1 || (G != 64 && G != 128) || (fmt != 2 && fmt != 3) || K % kLsSliceCols != 0 ||
        K > 8 * kLsSliceCols || N < 1)
        return cudaErrorNotSupported;
    const bool wide = G == 128 || fmt == 2;
    const uintptr_t ca = reinterpret_cast<uintptr_t>(codes), sa = reinterpret_cast<uintptr_t>(scales);
    if ((ca & (wide ? 7 : 3)) || (sa & (G == 128 ? 7 : 15))) return cudaErrorNotSupported;
    LsArgs a{};
    a.X = X;
    a.codes = codes;
    a.scales = scales;
    a.N = N;
    a.K = (int)K;
    a.CS = (int)(K / kLsSliceCols);
    a.Y = Y;
    a.y_bf16 = y_bf16;
    a.d_err = d_err;
    if (fmt == 2) return G == 128 ? launch_ls_cs<128, 2>(a, stream, sm_count) : launch_ls_cs<64, 2>(a, stream, sm_count);
    return G == 128 ? launch_ls_cs<128, 3>(a, stream, sm_count) : launch_ls_cs<64, 3>(a, stream, sm_count);
}

// The affine 4-bit codes (uint32 [N][K/8], low nibble first) with bf16 scales
// and biases [N][K/G].  Returns cudaErrorNotSupported when the shape is not
// covered: M != 1, G not 64 or 128, K not a multiple of 256 or above 2048,
// codes not 8-byte aligned, scales or biases not aligned to G = 128 ? 4 : 8.
cudaError_t launch_gemv_lut_stream_w4(const uint16_t* X, int64_t M, const uint32_t* codes, const uint16_t* scales,
                                      const uint16_t* biases, int64_t N, int64_t K, int G, void* Y, int y_bf16,
                                      cudaStream_t stream, int sm_count) {
    constexpr int SC = ls_slice_cols<4>();
    if (M != 1 || (G != 64 && G != 128) || K % SC != 0 || K > 8 * SC || N < 1) return cudaErrorNotSupported;
    const uintptr_t ca = reinterpret_cast<uintptr_t>(codes), sa = reinterpret_cast<uintptr_t>(scales),
                    ba = reinterpret_cast<uintptr_t>(biases);
    const uintptr_t sm = G == 128 ? 3 : 7;
    if ((ca & 7) || (sa & sm) || (ba & sm)) return cudaErrorNotSupported;
    LsArgs a{};
    a.X = X;
    a.codes = reinterpret_cast<const uint8_t*>(codes);
    a.scales = scales;
    a.biases = biases;
    a.N = N;
    a.K = (int)K;
    a.CS = (int)(K / SC);
    a.Y = Y;
    a.y_bf16 = y_bf16;
    a.d_err = nullptr;
    return G == 128 ? launch_ls_cs<128, 4>(a, stream, sm_count) : launch_ls_cs<64, 4>(a, stream, sm_count);
}

}  // namespace tq
