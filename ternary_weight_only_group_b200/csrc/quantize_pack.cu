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

// One lane per group (G = 8, 16, 32, 64, 128): the group's weights sit in
// the lane's registers (G = 128: one half at a time, read twice), so max and
// sum need no shuffles; every weight's byte
// and power of three are compile-time constants, so encoding is one
// multiply-add per weight into packed code words; each warp's 32 groups of
// code bytes are assembled in shared memory and written with 16-byte stores
// when the destination allows it.  The scale arithmetic is the one above.
// FMT selects the packing: 3 = base-3 (five digits per byte), 2 = the 2-bit
// format (four codes per byte; these G are multiples of 4, no padding).
template <int G, int FMT = 3>
__global__ void __launch_bounds__(256, G <= 32 ? 3 : 2) quantize_pack_group_kernel(
    const uint16_t* __restrict__ W, int64_t num_groups, uint8_t* __restrict__ codes,
    uint16_t* __restrict__ scales, uint32_t* __restrict__ d_err) {
    constexpr int NWD = G / 2;                 // 32-bit words of a group
    constexpr int PER = FMT == 3 ? 5 : 4;  // codes per byte
    constexpr int B = (G + PER - 1) / PER;
    constexpr int NCW = (B + 3) / 4;           // packed code words
    __shared__ __align__(16) uint8_t stage[256 / 32][32 * B];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const bool vec_out = (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
    uint32_t err_acc = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // The warp's next 32 groups (G <= 64) or next half-groups of 64 weights
    // (G = 128) are copied into a double-buffered shared-memory ring by
    // coalesced cp.async while the current ones are quantized (the loads cost
    // no registers, which the group occupies).  Ring rows are padded to
    // 16 bytes past the data so that the 16-byte reads of the lanes' own rows
    // are free of bank conflicts.
    constexpr int RS = (G <= 64 ? 2 * G : 128) + 16;
    extern __shared__ __align__(16) uint8_t qring[];  // [2][8 warps][32 rows][RS]
    auto issue = [&](int64_t gb, int half, int buf) {
        constexpr int PIECES = (G <= 64 ? G : 64) / 8;  // 16-byte pieces of a ring row
        uint8_t* base = qring + ((size_t)buf * 8 + wib) * 32 * RS;
#pragma unroll
        for (int k = 0; k < PIECES; ++k) {
            const int c = lane + 32 * k, grp = c / PIECES, piece = c - grp * PIECES;
            if (gb + grp < num_groups)
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                                 (uint32_t)__cvta_generic_to_shared(base + grp * RS + piece * 16)),
                             "l"(__cvta_generic_to_global(W + (gb + grp) * G + half * 64 + piece * 8))
                             : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // Waits for the oldest copy group in flight and reads this lane's ring row.
    auto take = [&](int buf, uint32_t* h) {
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncwarp();
        const uint4* row = reinterpret_cast<const uint4*>(qring + (((size_t)buf * 8 + wib) * 32 + lane) * RS);
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
    if (g_first < num_groups) issue(g_first, 0, 0);
    int pass = 0;
    for (int64_t g0 = g_first; g0 < num_groups; g0 += stride, ++pass) {
        const int64_t gi = g0 + lane;  // the warp's groups g0 .. g0+31
        const bool active = gi < num_groups;
        uint16_t s = 0;
        uint32_t gerr = 0;
        uint32_t cw[NCW];
        if constexpr (G <= 64) {
            uint32_t h[NWD];
            issue(g0 + stride, 0, (pass + 1) & 1);  // that buffer was read last pass
            take(pass & 1, h);
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
            if (gerr) s = 0;
            const uint32_t th = trit_threshold(s);
            // code words: byte q of the group in byte q % 4 of word q / 4; code
            // d = t + 1 of weight j at code_place(j); positions j >= G hold the
            // padding code 1
#pragma unroll
            for (int i = 0; i < NCW; ++i) cw[i] = 0;
#pragma unroll
            for (int j = 0; j < PER * B; ++j) {
                const uint32_t pw = code_place<FMT>(j);
                if (j < G) {
                    const uint32_t hw = h[j >> 1] >> (16 * (j & 1));
                    const uint32_t d = ((hw & 0x7FFFu) > th) ? ((hw & 0x8000u) ? 0u : 2u) : 1u;
                    cw[j / PER / 4] += d * pw;
                } else {
                    cw[j / PER / 4] += pw;  // padding code 1
                }
            }
        } else {
            // G = 128: the group is read twice in halves of 64 weights, so only
            // one half (32 words) is live at a time.  Pass 1 takes max, the
            // smallest nonzero magnitude and the binary64 sum of every nonzero
            // magnitude; the sum is exact when all of them lie within 2^37 of the
            // maximum (the same window as above), else the group takes the exact
            // multi-word path.  Pass 2 re-reads the halves (cache hits) to encode.
            // Ring steps: half 0 and 1 of pass 1 in buffers 0 and 1, then of
            // pass 2; each step issues the next (the last one the next 32
            // groups' first half).
            uint32_t amax = 0, amin1 = 0xFFFFFFFFu;  // amin1 = smallest nonzero magnitude - 1
            double sum = 0.0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t h[32];
                issue(g0, 1 - half, 1 - half);
                take(half, h);
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const uint32_t a = (h[j >> 1] >> (16 * (j & 1))) & 0x7FFFu;
                    amax = max(amax, a);
                    amin1 = min(amin1, a - 1u);  // a = 0 wraps to the largest value
                    if (a) sum += bf16_normal_mag_to_f64(a);
                }
            }
            const uint32_t emax = amax >> 7;
            const uint32_t thr = emax > 37 ? (emax - 37) << 7 : 0;
            const bool outside = amin1 != 0xFFFFFFFFu && amin1 + 1u < thr;
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
            if (gerr) s = 0;
            const uint32_t th = trit_threshold(s);
#pragma unroll
            for (int i = 0; i < NCW; ++i) cw[i] = 0;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t h[32];
                issue(half == 0 ? g0 : g0 + stride, 1 - half, 1 - half);
                take(half, h);
#pragma unroll
                for (int jj = 0; jj < 64; ++jj) {
                    const int j = 64 * half + jj;
                    const uint32_t hw = h[jj >> 1] >> (16 * (jj & 1));
                    const uint32_t d = ((hw & 0x7FFFu) > th) ? ((hw & 0x8000u) ? 0u : 2u) : 1u;
                    cw[j / PER / 4] += d * code_place<FMT>(j);
                }
            }
#pragma unroll
            for (int j = G; j < PER * B; ++j) cw[j / PER / 4] += code_place<FMT>(j);  // padding codes 1
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
static size_t quantize_ring_bytes(int G) { return (size_t)2 * 8 * 32 * ((G <= 64 ? 2 * G : 128) + 16); }

template <int G, int FMT = 3>
static cudaError_t launch_quantize_group(const uint16_t* W, int64_t num_groups, uint8_t* codes, uint16_t* scales,
                                         uint32_t* d_err, cudaStream_t stream, int grid) {
    auto kern = quantize_pack_group_kernel<G, FMT>;
    const size_t smem = quantize_ring_bytes(G);
    static SmemAttr smem_attr;
    if ((int)smem > 48 * 1024)
        if (cudaError_t e = smem_attr.ensure(kern, (int)smem)) return e;
    kern<<<grid, 256, smem, stream>>>(W, num_groups, codes, scales, d_err);
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
                                         grid_for((num_groups + 31) / 32 * 32, block, sm_count));
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
        case 8: return launch_quantize_group<8, 2>(W, num_groups, codes, scales, d_err, stream, grid);
        case 16: return launch_quantize_group<16, 2>(W, num_groups, codes, scales, d_err, stream, grid);
        case 32: return launch_quantize_group<32, 2>(W, num_groups, codes, scales, d_err, stream, grid);
        case 64: return launch_quantize_group<64, 2>(W, num_groups, codes, scales, d_err, stream, grid);
        case 128: return launch_quantize_group<128, 2>(W, num_groups, codes, scales, d_err, stream, grid);
        default: break;
    }
    quantize_pack2_generic_kernel<<<grid_for(num_groups, 128, sm_count), 128, 0, stream>>>(
        W, num_groups, G, codes, scales, d_err);
    return cudaGetLastError();
}

}  // namespace tq
