// quantize_pack.cu -- per-group ternary quantizer and base-3 packer.
//
// "precisit/pack-unpack-run", codec.py description: each group's scale is
// the mean of |w| stored as fp16; trits come from rounding w / scale half to
// even; five trits go into a byte as base-3 digits; every group starts on a
// byte boundary and unused digit slots hold the zero trit.
//
// The matrix is treated as a flat run of N*K/G groups (a group never crosses
// a row because K % G == 0).  Fast path (G = 8 * 2^k, 8 <= G <= 256): a warp
// covers 32*8/G consecutive groups, G/8 lanes per group, 8 weights per lane
// from one 16-byte load; the group's max |w| and sum |w| are segmented warp
// shuffle reductions.  The sum is exact: every |w| within 2^37 of the group
// maximum fits, together with the total, in the 53-bit binary64 significand,
// so the shuffle order cannot change it; dividing by G (a power of two) is
// exact and cvt.rn.f16.f64 rounds once, ties to even.  A group holding a
// nonzero |w| more than 2^37 below its maximum takes the multi-word exact
// path instead.  Each lane loads the next pass's weights before it computes
// the current pass.  Other G use one thread per group with the multi-word
// path.
#include <atomic>

#include "tq_internal.cuh"

namespace tq {

template <int G>
__global__ void __launch_bounds__(256) quantize_pack_pow2_kernel(
    const uint16_t* __restrict__ W, int64_t num_groups, uint8_t* __restrict__ codes,
    uint16_t* __restrict__ scales, uint32_t* __restrict__ d_err) {
    constexpr int LPG = G / 8;     // lanes per group
    constexpr int GPW = 32 / LPG;  // groups per warp pass
    constexpr int B = bytes_per_group(G);
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPG;
    const int p0 = 8 * sub;  // first weight of this lane inside its group
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    uint32_t err_acc = 0;

    // The next pass's 16-byte load is issued before this pass is computed
    // (two loads in flight per lane).
    const int64_t stride = nwarps * GPW;
    auto load = [&](int64_t base) {
        const int64_t gi = base + lane / LPG;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (gi < num_groups) v = __ldcs(reinterpret_cast<const uint4*>(W + gi * G + p0));
        return v;
    };
    uint4 v_next = load(warp * GPW);
    for (int64_t base = warp * GPW; base < num_groups; base += stride) {
        const int64_t gi = base + lane / LPG;
        const bool active = gi < num_groups;
        const uint4 v = v_next;
        v_next = load(base + stride);
        const uint32_t h[4] = {v.x, v.y, v.z, v.w};
        uint32_t a[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[2 * i] = h[i] & 0x7FFFu;
            a[2 * i + 1] = (h[i] >> 16) & 0x7FFFu;
        }
        uint32_t amax = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = max(amax, a[i]);
        amax = seg_max_u32(amax, LPG);  // NaN/Inf patterns are the largest magnitudes

        // All 32 lanes run every shuffle below; the per-group decisions come after.
        const uint32_t emax = amax >> 7;
        const uint32_t thr = emax > 37 ? (emax - 37) << 7 : 0;  // smallest pattern in the window
        double sum = 0.0;
        uint32_t outside = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (a[i] >= thr) sum += bf16_normal_mag_to_f64(a[i]);
            else outside |= a[i];
        }
        sum = seg_sum_f64(sum, LPG);
        outside = seg_or_u32(outside, LPG);

        uint16_t s = 0;
        uint32_t gerr = 0;
        bool slow = false;
        if (amax >= 0x7F80u) {
            gerr = TQ_DERR_WEIGHT;
        } else if (amax > kTinyMaxBits) {
            if (outside) {
                slow = true;
            } else {
                const uint16_t bits = __half_as_ushort(__double2half(sum * (1.0 / G)));
                if (bits >= 0x7C00u) gerr = TQ_DERR_OVERFLOW;
                else s = bits;
            }
        }
        if (__any_sync(0xffffffffu, slow)) {
            if (slow && sub == 0 && active) gerr = exact_group_scale(W + gi * G, G, &s);
            const int leader = lane - sub;  // same value for every lane of a segment
            s = (uint16_t)__shfl_sync(0xffffffffu, (uint32_t)s, leader, 32);
            gerr = __shfl_sync(0xffffffffu, gerr, leader, 32);
        }
        if (gerr) s = 0;

        // digits d = t + 1 of this lane's 8 weights, 2 bits each
        const uint32_t th = trit_threshold(s);
        uint32_t F = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const uint32_t hw = (h[i] >> (16 * k)) & 0xFFFFu;
                const uint32_t d = (a[2 * i + k] > th) ? ((hw & 0x8000u) ? 0u : 2u) : 1u;
                F |= d << (2 * (2 * i + k));
            }
        }
        uint32_t Fn = __shfl_down_sync(0xffffffffu, F, 1);
        if (sub == LPG - 1) Fn = 0x5555u;  // positions >= G: padding digit 1
        const uint32_t D = F | (Fn << 16);  // digits of weights p0 .. p0+15

        if (active) {
            uint8_t* out = codes + gi * B;
            for (int q = (p0 + 4) / 5; 5 * q < p0 + 8 && q < B; ++q) {
                const uint32_t f = D >> (2 * (5 * q - p0));
                const uint32_t byte = (f & 3u) + 3u * ((f >> 2) & 3u) + 9u * ((f >> 4) & 3u) +
                                      27u * ((f >> 6) & 3u) + 81u * ((f >> 8) & 3u);
                out[q] = (uint8_t)byte;
            }
            if (sub == 0) {
                scales[gi] = s;
                err_acc |= gerr;
            }
        }
    }
    // Stores visible device-wide before the block exits: a matmul launched next on
    // the stream may read codes and scales before its grid-dependency wait.
    __threadfence();
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

// Place of weight j's code inside the group's packed words: code c of weight
// j adds c * code_place(j) to word (j / PER) / 4, PER codes per byte.  Base-3
// (FMT 3): digit j % 5 of byte j / 5, weight 3^(j % 5).  2-bit (FMT 2): bits
// 2 (j % 4) of byte j / 4.
template <int FMT>
__host__ __device__ constexpr uint32_t code_place(int j) {
    return (FMT == 3 ? (j % 5 == 0 ? 1u : j % 5 == 1 ? 3u : j % 5 == 2 ? 9u : j % 5 == 3 ? 27u : 81u)
                     : 1u << (2 * (j % 4)))
           << (8 * ((j / (FMT == 3 ? 5 : 4)) % 4));
}

// |w| of the two bf16 weights of a word as a pair of fp32 values (exact).
__device__ __forceinline__ uint64_t mag_pair_f32x2(uint32_t w) {
    return f2_pack(__uint_as_float((w << 16) & 0x7FFF0000u), __uint_as_float(w & 0x7FFF0000u));
}

// Sum of the G magnitudes of a group in fp32, the words' pairs spread over
// NA packed accumulators (2 NA chains; chain c adds the magnitudes of words
// i = c / 2 mod NA in order).  Recursive summation of nonnegative terms errs
// by at most (n - 1) u of the exact sum for a chain of n terms (u = 2^-24),
// and adding the 2 NA chains pairwise adds at most log2(2 NA) u more.
template <int NA, int NW>
__device__ __forceinline__ float group_sum_f32(const uint32_t (&h)[NW]) {
    uint64_t acc[NA];
#pragma unroll
    for (int a = 0; a < NA; ++a) acc[a] = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) acc[i % NA] = f2_add(acc[i % NA], mag_pair_f32x2(h[i]));
#pragma unroll
    for (int n = NA / 2; n >= 1; n >>= 1)
#pragma unroll
        for (int a = 0; a < n; ++a) acc[a] = f2_add(acc[a], acc[a + n]);
    const float2 r = f2_unpack(acc[0]);
    return r.x + r.y;
}

// RNE_fp16(mean |w|) from a computed sum S of the G magnitudes whose relative
// error is at most rel: accepted when S is finite and both ends of
// [S (1 - rel), S (1 + rel)] / G round to the same finite binary16 (the
// exact mean lies between them and rounding is monotone; the endpoints are
// formed in binary64, whose own rounding is far inside the slack in rel).
// Otherwise the caller takes an exact path: a mean within rel of a rounding
// tie, a rejected (Inf/NaN) weight, or an overflowing mean.
template <int G>
__device__ __forceinline__ bool scale_from_sum(double S, double rel, uint16_t* s) {
    if (!(S <= 3.4028234663852886e38)) return false;  // Inf or NaN
    const double m = S * (1.0 / G);
    const uint16_t lo = __half_as_ushort(__double2half(m * (1.0 - rel)));
    const uint16_t hi = __half_as_ushort(__double2half(m * (1.0 + rel)));
    if (lo != hi || lo >= 0x7C00u) return false;
    *s = lo;
    return true;
}

// Codes d = t + 1 (0, 1, 2) of the two bf16 weights of a word, in the two
// 16-bit halves: 2 where w > s/2, 0 where w < -s/2, else 1 (ties round to
// the even trit 0).  thp holds th = floor_bf16(s / 2) in both halves, thn
// -th; for s = 0 both are NaN patterns and every code is 1.  A bf16 weight
// exceeds s/2 exactly when it exceeds th.
__device__ __forceinline__ uint32_t codes_pair(uint32_t w, uint32_t thp, uint32_t thn) {
    uint32_t g, l;
    asm("set.gt.u32.bf16x2 %0, %1, %2;" : "=r"(g) : "r"(w), "r"(thp));
    asm("set.lt.u32.bf16x2 %0, %1, %2;" : "=r"(l) : "r"(w), "r"(thn));
    return 0x00010001u + (g & 0x00010001u) - (l & 0x00010001u);
}

// Packed code words of a group from its words' code pairs, in word order:
// byte q is the sum over its weights j of code_j * place_j (3^(j mod 5)
// base-3, 4^(j mod 4) 2-bit), and the 4 bytes of a packed word cover exactly
// WPW = 2 PER words of weights.  a[r] collects byte 4k + r of the current
// packed word k in bits 16..31: a pair d2 = lo + 2^16 hi times (Q + 2^16 P)
// leaves lo P + hi Q there (P, Q the places of the pair's weights in that
// byte, 0 for a weight of another byte), while the lo Q products below stay
// under 2^16.  Padding positions (j >= G) add their code 1.  Only the four
// accumulators of the word being built are live.
template <int G, int FMT>
struct CodeWords {
    static constexpr int PER = FMT == 3 ? 5 : 4;
    static constexpr int B = (G + PER - 1) / PER;
    static constexpr int NCW = (B + 3) / 4;
    static constexpr int NWD = G / 2;
    static constexpr int WPW = 2 * PER;
    uint32_t a[4];
    static __host__ __device__ constexpr uint32_t place(int j) {
        return FMT == 3 ? (j % 5 == 0 ? 1u : j % 5 == 1 ? 3u : j % 5 == 2 ? 9u : j % 5 == 3 ? 27u : 81u)
                        : 1u << (2 * (j % 4));
    }
    static __host__ __device__ constexpr uint32_t padding(int q) {
        uint32_t pad = 0;
        for (int j = PER * q; j < PER * q + PER; ++j)
            if (j >= G) pad += place(j);
        return pad << 16;
    }
    // word i of the group (weights 2i, 2i + 1), i = 0 .. NWD - 1 in order
    __device__ __forceinline__ void put(int i, uint32_t d2, uint32_t (&cw)[NCW]) {
        const int k = i / WPW;
        if (i % WPW == 0) {
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = padding(4 * k + r);
        }
        const int j0 = 2 * i, j1 = 2 * i + 1, r0 = j0 / PER - 4 * k, r1 = j1 / PER - 4 * k;
        if (r0 == r1) {
            a[r0] += d2 * (place(j1) + (place(j0) << 16));
        } else {
            a[r0] += d2 * (place(j0) << 16);
            a[r1] += d2 * place(j1);
        }
        if (i % WPW == WPW - 1 || i == NWD - 1) {
            const uint32_t b1 = 4 * k + 1 < B ? a[1] : 0u, b2 = 4 * k + 2 < B ? a[2] : 0u,
                           b3 = 4 * k + 3 < B ? a[3] : 0u;
            cw[k] = prmt32(prmt32(a[0], b1, 0x0062u), prmt32(b2, b3, 0x0062u), 0x5410u);
        }
    }
};

// One lane per group (G = 8, 16, 32, 64, 128): the group's weights sit in
// the lane's registers, so sum and codes need no shuffles.  The scale comes
// from an fp32 sum of the magnitudes (packed pairs, several chains) checked
// against its error bound (scale_from_sum); the rare group near a rounding
// tie takes the exact binary64 window of the fast path above, or the
// multi-word path.  Codes: two bf16 comparisons per pair of weights
// (codes_pair) and one multiply-add per pair into the current packed word
// (CodeWords), every place value a compile-time constant.  Each warp's 32
// groups of code bytes are assembled in shared memory and written with
// 16-byte stores when the destination allows it.  FMT selects the packing:
// 3 = base-3 (five digits per byte), 2 = the 2-bit format (four codes per
// byte; these G are multiples of 4, no padding).
// Threads per block of the group kernel: G = 128 holds its whole group (64
// words) in registers and its ring rows are 272 bytes, so it runs 128-thread
// blocks, three per SM; the others 256.
template <int G>
constexpr int qg_threads() { return G == 128 ? 128 : 256; }

template <int G, int FMT = 3>
__global__ void __launch_bounds__(qg_threads<G>(), G <= 32 || G == 128 ? 3 : 2) quantize_pack_group_kernel(
    const uint16_t* __restrict__ W, int64_t num_groups, uint8_t* __restrict__ codes,
    uint16_t* __restrict__ scales, uint32_t* __restrict__ d_err) {
    constexpr int NWD = G / 2;                 // 32-bit words of a group
    constexpr int PER = FMT == 3 ? 5 : 4;  // codes per byte
    constexpr int B = (G + PER - 1) / PER;
    constexpr int NCW = (B + 3) / 4;           // packed code words
    constexpr int NW = qg_threads<G>() / 32;  // warps per block
    __shared__ __align__(16) uint8_t stage[NW][32 * B];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const bool vec_out = (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
    uint32_t err_acc = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // The warp's next 32 groups are copied into a double-buffered
    // shared-memory ring by coalesced cp.async while the current ones are
    // quantized (the loads cost no registers, which the group occupies).  Ring
    // rows are padded to 16 bytes past the data so that the 16-byte reads of
    // the lanes' own rows are free of bank conflicts.
    constexpr int RS = 2 * G + 16;
    extern __shared__ __align__(16) uint8_t qring[];  // [2][NW warps][32 rows][RS]
    auto issue = [&](int64_t gb, int buf) {
        constexpr int PIECES = G / 8;  // 16-byte pieces of a ring row
        uint8_t* base = qring + ((size_t)buf * NW + wib) * 32 * RS;
#pragma unroll
        for (int k = 0; k < PIECES; ++k) {
            const int c = lane + 32 * k, grp = c / PIECES, piece = c - grp * PIECES;
            if (gb + grp < num_groups)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                                 (uint32_t)__cvta_generic_to_shared(base + grp * RS + piece * 16)),
                             "l"(__cvta_generic_to_global(W + (gb + grp) * G + piece * 8))
                             : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // Waits for the oldest copy group in flight and reads this lane's ring row.
    auto take = [&](int buf, uint32_t* h) {
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncwarp();
        const uint4* row = reinterpret_cast<const uint4*>(qring + (((size_t)buf * NW + wib) * 32 + lane) * RS);
#pragma unroll
        for (int k = 0; k < (RS - 16) / 16; ++k) {
            const uint4 v = row[k];
            h[4 * k] = v.x;
            h[4 * k + 1] = v.y;
            h[4 * k + 2] = v.z;
            h[4 * k + 3] = v.w;
        }
        __syncwarp();  // every lane has read this buffer before it is refilled
    };
    const int64_t g_first = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
    if (g_first < num_groups) issue(g_first, 0);
    int pass = 0;
    for (int64_t g0 = g_first; g0 < num_groups; g0 += stride, ++pass) {
        const int64_t gi = g0 + lane;  // the warp's groups g0 .. g0+31
        const bool active = gi < num_groups;
        uint16_t s = 0;
        uint32_t gerr = 0;
        uint32_t cw[NCW];
        {
            uint32_t h[NWD];
            issue(g0 + stride, (pass + 1) & 1);  // that buffer was read last pass
            take(pass & 1, h);
            // fp32 sum in 8 chains of G / 16 terms (G = 8..64; 16 chains of 8 at
            // G = 128); a group whose mean lies within the sum's error of a
            // rounding tie, or that holds an Inf/NaN weight or overflows, takes
            // the exact binary64 window below
            constexpr int NA = G == 128 ? 8 : NWD >= 4 ? 4 : NWD;
            constexpr int TPC = (NWD + NA - 1) / NA;  // terms per chain
            if (!scale_from_sum<G>((double)group_sum_f32<NA>(h), (TPC + 4) * 0x1p-24, &s)) {
                uint32_t amax = 0;
#pragma unroll
                for (int j = 0; j < G; ++j) amax = max(amax, (h[j >> 1] >> (16 * (j & 1))) & 0x7FFFu);
                const uint32_t emax = amax >> 7;
                const uint32_t thr = emax > 37 ? (emax - 37) << 7 : 0;  // smallest pattern in the exact window
                double sum = 0.0;
                uint32_t outside = 0;
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    const uint32_t a = (h[j >> 1] >> (16 * (j & 1))) & 0x7FFFu;
                    if (a >= thr) sum += bf16_normal_mag_to_f64(a);
                    else outside |= a;
                }
                if (amax >= 0x7F80u) {
                    gerr = TQ_DERR_WEIGHT;
                } else if (amax > kTinyMaxBits) {
                    if (outside) {
                        gerr = exact_group_scale(W + (active ? gi : 0) * G, G, &s);
                    } else {
                        const uint16_t bits = __half_as_ushort(__double2half(sum * (1.0 / G)));
                        if (bits >= 0x7C00u) gerr = TQ_DERR_OVERFLOW;
                        else s = bits;
                    }
                }
            }
            if (gerr) s = 0;
            const uint32_t th = trit_threshold(s);
            const uint32_t thp = th | (th << 16), thn = thp | 0x80008000u;
            CodeWords<G, FMT> cwb;
#pragma unroll
            for (int i = 0; i < NWD; ++i) cwb.put(i, codes_pair(h[i], thp, thn), cw);
        }
        if (active) {
            scales[gi] = s;
            err_acc |= gerr;
        }
        // the warp's 32 * B code bytes, contiguous from g0 * B
        uint8_t* st = stage[wib] + lane * B;
#pragma unroll
        for (int q = 0; q < B; ++q) st[q] = (uint8_t)(cw[q / 4] >> (8 * (q % 4)));
        __syncwarp();
        const int64_t nvalid = (num_groups - g0 < 32 ? num_groups - g0 : 32) * B;
        uint8_t* out = codes + g0 * B;
        if (vec_out && nvalid == 32 * B) {  // 32 * B is a multiple of 16 for these G
            for (int c = lane; c < 2 * B; c += 32)
                reinterpret_cast<uint4*>(out)[c] = reinterpret_cast<const uint4*>(stage[wib])[c];
        } else {
            for (int c = lane; c < nvalid; c += 32) out[c] = stage[wib][c];
        }
        __syncwarp();
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // Stores visible device-wide before the block exits: a matmul launched next on
    // the stream may read codes and scales before its grid-dependency wait.
    __threadfence();
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

// Dynamic shared memory of quantize_pack_group_kernel: the load ring.
static size_t quantize_ring_bytes(int G) { return (size_t)2 * (G == 128 ? 4 : 8) * 32 * (2 * G + 16); }

template <int G, int FMT = 3>
static cudaError_t launch_quantize_group(const uint16_t* W, int64_t num_groups, uint8_t* codes, uint16_t* scales,
                                         uint32_t* d_err, cudaStream_t stream, int grid, int sm_count) {
    auto kern = quantize_pack_group_kernel<G, FMT>;
    const size_t smem = quantize_ring_bytes(G);
    static SmemAttr smem_attr;
    if ((int)smem > 48 * 1024)
        if (cudaError_t e = smem_attr.ensure(kern, (int)smem)) return e;
    // one wave of resident blocks, each warp looping over many passes: the
    // ring's fill is paid once per warp, and a warp that takes the slow exact
    // path delays only itself, not the tail of a wave of short blocks
    static std::atomic<int> per_sm{0};
    int bps = per_sm.load();
    if (bps == 0) {
        if (cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, kern, qg_threads<G>(), smem)) return e;
        bps = bps < 1 ? 1 : bps;
        per_sm.store(bps);
    }
    if (grid > bps * sm_count) grid = bps * sm_count;
    kern<<<grid, qg_threads<G>(), smem, stream>>>(W, num_groups, codes, scales, d_err);
    return cudaGetLastError();
}

// Any G: one thread per group, multi-word exact scale.
__global__ void __launch_bounds__(128) quantize_pack_generic_kernel(
    const uint16_t* __restrict__ W, int64_t num_groups, int G, uint8_t* __restrict__ codes,
    uint16_t* __restrict__ scales, uint32_t* __restrict__ d_err) {
    const int B = bytes_per_group(G);
    uint32_t err_acc = 0;
    for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < num_groups;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const uint16_t* w = W + gi * G;
        uint16_t s;
        const uint32_t gerr = exact_group_scale(w, G, &s);
        err_acc |= gerr;
        scales[gi] = s;
        const uint32_t th = trit_threshold(s);
        uint8_t* out = codes + gi * B;
        for (int q = 0; q < B; ++q) {
            uint32_t byte = 0, p3 = 1;
            for (int i = 0; i < 5; ++i) {
                const int j = 5 * q + i;
                uint32_t d = 1;
                if (j < G) {
                    const uint32_t hw = w[j];
                    d = ((hw & 0x7FFFu) > th) ? ((hw & 0x8000u) ? 0u : 2u) : 1u;
                }
                byte += d * p3;
                p3 *= 3;
            }
            out[q] = (uint8_t)byte;
        }
    }
    // Stores visible device-wide before the block exits: a matmul launched next on
    // the stream may read codes and scales before its grid-dependency wait.
    __threadfence();
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

static int grid_for(int64_t threads_needed, int block, int sm_count) {
    int64_t blocks = (threads_needed + block - 1) / block;
    const int64_t cap = (int64_t)sm_count * 16;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

cudaError_t launch_quantize_pack(const uint16_t* W, int64_t N, int64_t K, int G, uint8_t* codes,
                                 uint16_t* scales, uint32_t* d_err, cudaStream_t stream,
                                 int sm_count) {
    const int64_t num_groups = N * (K / G);
    if (num_groups == 0) return cudaSuccess;
    const int block = 256;
#define TQ_QP_CASE(GG)                                                                           \
    case GG: {                                                                                   \
        const int64_t threads = (num_groups + (32 / (GG / 8)) - 1) / (32 / (GG / 8)) * 32;       \
        quantize_pack_pow2_kernel<GG><<<grid_for(threads, block, sm_count), block, 0, stream>>>( \
            W, num_groups, codes, scales, d_err);                                                \
        return cudaGetLastError();                                                               \
    }
#define TQ_QG_CASE(GG)                                                                              \
    case GG:                                                                                        \
        return launch_quantize_group<GG>(W, num_groups, codes, scales, d_err, stream,              \
                                         grid_for((num_groups + 31) / 32 * 32, block, sm_count), sm_count);
    switch (G) {
        TQ_QG_CASE(8)
        TQ_QG_CASE(16)
        TQ_QG_CASE(32)
        TQ_QG_CASE(64)
        TQ_QG_CASE(128)
        TQ_QP_CASE(256)
        default:
            break;
    }
#undef TQ_QP_CASE
#undef TQ_QG_CASE
    quantize_pack_generic_kernel<<<grid_for(num_groups, 128, sm_count), 128, 0, stream>>>(
        W, num_groups, G, codes, scales, d_err);
    return cudaGetLastError();
}

// 2-bit format, any G: one thread per group, multi-word exact scale; code
// t + 1 of weight j in bits 2 (j % 4) of byte j / 4, padding codes 1.
__global__ void __launch_bounds__(128) quantize_pack2_generic_kernel(
    const uint16_t* __restrict__ W, int64_t num_groups, int G, uint8_t* __restrict__ codes,
    uint16_t* __restrict__ scales, uint32_t* __restrict__ d_err) {
    const int B = (G + 3) / 4;
    uint32_t err_acc = 0;
    for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < num_groups;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const uint16_t* w = W + gi * G;
        uint16_t s;
        const uint32_t gerr = exact_group_scale(w, G, &s);
        err_acc |= gerr;
        scales[gi] = s;
        const uint32_t th = trit_threshold(s);
        uint8_t* out = codes + gi * B;
        for (int q = 0; q < B; ++q) {
            uint32_t byte = 0;
            for (int i = 0; i < 4; ++i) {
                const int j = 4 * q + i;
                uint32_t d = 1;
                if (j < G) {
                    const uint32_t hw = w[j];
                    d = ((hw & 0x7FFFu) > th) ? ((hw & 0x8000u) ? 0u : 2u) : 1u;
                }
                byte |= d << (2 * i);
            }
            out[q] = (uint8_t)byte;
        }
    }
    // Stores visible device-wide before the block exits: a matmul launched next on
    // the stream may read codes and scales before its grid-dependency wait.
    __threadfence();
    if (err_acc && d_err) atomicOr(d_err, err_acc);
}

cudaError_t launch_quantize_pack2(const uint16_t* W, int64_t N, int64_t K, int G, uint8_t* codes,
                                  uint16_t* scales, uint32_t* d_err, cudaStream_t stream, int sm_count) {
    const int64_t num_groups = N * (K / G);
    if (num_groups == 0) return cudaSuccess;
    const int grid = grid_for((num_groups + 31) / 32 * 32, 256, sm_count);
    switch (G) {
        case 8: return launch_quantize_group<8, 2>(W, num_groups, codes, scales, d_err, stream, grid, sm_count);
        case 16: return launch_quantize_group<16, 2>(W, num_groups, codes, scales, d_err, stream, grid, sm_count);
        case 32: return launch_quantize_group<32, 2>(W, num_groups, codes, scales, d_err, stream, grid, sm_count);
        case 64: return launch_quantize_group<64, 2>(W, num_groups, codes, scales, d_err, stream, grid, sm_count);
        case 128: return launch_quantize_group<128, 2>(W, num_groups, codes, scales, d_err, stream, grid, sm_count);
        default: break;
    }
    quantize_pack2_generic_kernel<<<grid_for(num_groups, 128, sm_count), 128, 0, stream>>>(
        W, num_groups, G, codes, scales, d_err);
    return cudaGetLastError();
}

}  // namespace tq
