// gemv_lut.cu -- decode GEMV by activation lookup tables (CUDA cores, sm_100a).
//
// Computes the fused unpack-and-scale matmul of tiny-llm "Week 2 Day 3:
// Quantize the Model" ("Mathematical Formulation": C[i,k] = sum_g scale[k,g] *
// sum_j q[k,j] A[i,j], bias 0) for the ternary format of
// "precisit/pack-unpack-run" (codec.py: five base-3 digits per byte, each
// group byte-aligned).  Instead of decoding every weight, each code byte
// indexes a table of the 243 possible partial sums sum_i t_i x_i over the five
// activations it covers (the lookup-table GEMV idea): one shared-memory load
// and one FMA per byte, the FMA applying the group scale.
//
// Work decomposition (group sizes with 13- or 26-byte groups: G = 61..65 or
// 126..130; the common G = 64 and G = 128):
//   * 13 lanes cover one group, each owning BPL = B/13 consecutive code bytes;
//     a "slice" is two groups (26 lanes).  Lane l's tables live only in
//     shared-memory bank l, so a warp's lookups never conflict whatever the
//     code bytes are.
//   * A CTA owns R rows and, per pass, NS slices whose tables are resident;
//     the CS CTAs of a thread-block cluster split K and add their partial
//     rows through distributed shared memory in a fixed rank order.
//   * Warps take batches of 8 rows; per-row sums are formed by a transposing
//     butterfly so each lane ends with one row's total.
//   * Codes and scales do not depend on earlier kernels: they are requested
//     before griddepcontrol.wait, so under programmatic dependent launch the
//     weight traffic overlaps the previous kernel; activations are read after.
// Invalid bytes (>= 243), non-canonical padding and bad scales make table
// entries or scales NaN, so the affected row is NaN; such rows are rescanned
// to report the exact error bits.
#include <cooperative_groups.h>

#include <atomic>
#include <cstdio>
#include <cstdlib>

#include "tq_internal.cuh"

namespace cg = cooperative_groups;

namespace tq {

// CTA size: 256 threads (two CTAs per SM, so a dependent launch can start
// beside the running one) for small matrices, 512 for large ones.
constexpr int kRB = 8;                 // rows per warp batch
constexpr int kLPG = 13;               // lanes per group
constexpr int kGPS = 2;                // groups per slice
constexpr int kLanes = kLPG * kGPS;    // active lanes (26)
constexpr int kTableWords = 256 * 32;  // one chunk position of one slice: 256 entries x 32 banks

struct LutPlan {
    int S;        // slices per row
    int CS;       // CTAs per cluster (split of K)
    int NS;       // slices resident per pass
    int P;        // passes per CTA
    int R;        // rows per CTA
    int RP;       // R rounded up to 32: stride of the per-row shared arrays
    int RB;       // row blocks (grid = RB * CS)
    int MT;       // tokens per launch
    int PER;      // rows reduced by each cluster rank = ceil(R / CS)
    int THREADS;  // 256 (small matrices, two CTAs per SM) or 512
    size_t smem;
    size_t off_scale, off_acc, off_red;
};

struct LutArgs {
    const uint16_t* X;
    int M, m0;
    const uint8_t* codes;
    const uint16_t* scales;
    int64_t N;
    int K, G, ng;
    int64_t row_bytes;
    LutPlan p;
    void* Y;
    int y_bf16;
    uint32_t* d_err;
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// Decoded scale as used by the matmul: RNE_bf16(binary16 s) as fp32; NaN for a
// rejected scale so every output of its row is NaN.
__device__ __forceinline__ float decoded_scale(uint32_t s) {
    if (scale_is_bad(s)) return __uint_as_float(0x7FC00000u);
    return bf16_bits_to_f32(scale_to_bf16_bits((uint16_t)s));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

// Transposing butterfly: on entry every lane holds v[0..RB); on exit lane l
// (l < RB) holds the sum over all 32 lanes of v[l].
template <int RB>
__device__ __forceinline__ float transpose_reduce(float (&v)[RB]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o >= RB; o >>= 1) {
#pragma unroll
        for (int i = 0; i < RB; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
    }
#pragma unroll
    for (int n = RB / 2; n >= 1; n >>= 1) {  // n = half size, exchange distance n
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

// Writes the entries b = 81*d4 + [0, 81) of this lane's chunk table (d4 =
// part), or the 13 entries 243..255 (part == 3, always NaN).  With
// b = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4, entry(b) = P[d0 + 3 d1] + Q[d2 + 3 d3]
// where P and Q hold the partial sums sum_i (d_i - 1) x_i of their digits.  A
// digit position beyond G (the padding of a group's last byte) must hold 1:
// the P or Q terms that violate this are NaN, which makes every entry using
// them NaN at no per-entry cost.
template <int B>
__device__ __forceinline__ void build_part(const LutArgs& a, float* tab, int sl, int m, int j, int gg0,
                                           int part) {
    constexpr int BPL = B / kLPG;
    const int lane = threadIdx.x & 31;
    const int gl = lane / kLPG;
    const int q = (lane - gl * kLPG) * BPL + j;
    const float nan = __uint_as_float(0x7FC00000u);
    float* col = tab + lane;
    if (part == 3) {
#pragma unroll
        for (int b = 243; b < 256; ++b) col[b * 32] = nan;
        return;
    }
    float x[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    const int gg = gg0 + sl * kGPS + gl;
    const uint16_t* xr = a.X + (int64_t)(a.m0 + m) * a.K + (int64_t)gg * a.G + 5 * q;
    const int real = min(5, a.G - 5 * q);
#pragma unroll
    for (int i = 0; i < 5; ++i)
        if (i < real) x[i] = bf16_bits_to_f32(__ldcg(xr + i));  // written by the preceding kernel: bypass L1
    const int d4 = part;
    const bool bad4 = (4 >= real) && d4 != 1;
    const float h4 = (float)(d4 - 1) * x[4];
    float P[9], Q[9];
#pragma unroll
    for (int d3 = 0; d3 < 3; ++d3) {
#pragma unroll
        for (int d2 = 0; d2 < 3; ++d2) {
            const bool bad = bad4 || ((3 >= real) && d3 != 1) || ((2 >= real) && d2 != 1);
            const float v = h4 + (float)(d3 - 1) * x[3] + (float)(d2 - 1) * x[2];
            Q[d2 + 3 * d3] = bad ? nan : v;
        }
    }
#pragma unroll
    for (int d1 = 0; d1 < 3; ++d1) {
#pragma unroll
        for (int d0 = 0; d0 < 3; ++d0) {
            const bool bad = ((1 >= real) && d1 != 1) || ((0 >= real) && d0 != 1);
            const float v = (float)(d1 - 1) * x[1] + (float)(d0 - 1) * x[0];
            P[d0 + 3 * d1] = bad ? nan : v;
        }
    }
    float* c4 = col + 81 * 32 * d4;
#pragma unroll
    for (int i = 0; i < 9; ++i)
#pragma unroll
        for (int k = 0; k < 9; ++k) c4[(9 * i + k) * 32] = P[k] + Q[i];
}

template <int B, int MT, int NS, int kLutThreads>
__global__ void __launch_bounds__(kLutThreads, 512 / kLutThreads) gemv_lut_kernel(const LutArgs a) {
    constexpr int kLutWarps = kLutThreads / 32;
    constexpr int BPL = B / kLPG;
    constexpr int SLICE_BYTES = kGPS * B;
    extern __shared__ __align__(16) unsigned char smem[];
    float* table = reinterpret_cast<float*>(smem);
    const LutPlan& p = a.p;
    float* ssc = reinterpret_cast<float*>(smem + p.off_scale);  // [NS*GPS][RP] decoded scales
    float* acc_s = reinterpret_cast<float*>(smem + p.off_acc);  // [MT][RP] partial rows
    float* red = reinterpret_cast<float*>(smem + p.off_red);    // [CS][MT][PER] pushed partials

    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int rb = blockIdx.x / p.CS;
    const int64_t row0 = (int64_t)rb * p.R;
    const int nrows = (int)(a.N - row0 < (int64_t)p.R ? a.N - row0 : (int64_t)p.R);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool lane_on = lane < kLanes;
    const int g_local = lane_on ? lane / kLPG : 0;                     // inactive lanes read valid bytes
    const int qb = lane_on ? (lane - (lane / kLPG) * kLPG) * BPL : 0;  // first byte in the group
    const int nbatch = (nrows + kRB - 1) / kRB;
    const int ngl = NS * kGPS;
    const uint32_t table_s = smem_u32(table) + 4u * lane;
    const uint32_t ssc_s = smem_u32(ssc);

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    cluster_arrive_relaxed();  // waited on before the first store into a peer's shared memory

    for (int pass = 0; pass < p.P; ++pass) {
        const int gg0 = (crank * p.P + pass) * ngl;  // first group of this pass
        __syncthreads();  // previous pass finished with the tables and scales

        // code bytes of a batch of 8 rows x NS slices (rows past the end
        // repeat the last row; their sums are never stored)
        const uint8_t* cbase = a.codes + row0 * a.row_bytes + (int64_t)(gg0 + g_local) * B + qb;
        auto load_batch = [&](int bt, uint32_t (&cw)[NS][kRB]) {
            const int r0 = bt * kRB;
            const bool full = r0 + kRB <= nrows;
            const uint8_t* rp = cbase + (int64_t)r0 * a.row_bytes;
#pragma unroll
            for (int r = 0; r < kRB; ++r) {
                const int rr = full ? r : min(r, nrows - 1 - r0);
                const uint8_t* cp = rp + (uint32_t)rr * (uint32_t)a.row_bytes;
#pragma unroll
                for (int sl = 0; sl < NS; ++sl) {
                    if (BPL == 2)
                        cw[sl][r] = __ldg(reinterpret_cast<const uint16_t*>(cp + sl * SLICE_BYTES));
                    else
                        cw[sl][r] = __ldg(cp + sl * SLICE_BYTES);
                }
            }
        };
        auto run_batch = [&](int bt, const uint32_t (&cw)[NS][kRB]) {
            const int r0 = bt * kRB;
            float acc[MT][kRB];
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int r = 0; r < kRB; ++r) acc[m][r] = 0.f;
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) {
                const uint32_t sc = ssc_s + 4u * ((sl * kGPS + g_local) * p.RP + r0);
                const uint32_t tl = table_s + 4u * (sl * MT * BPL) * kTableWords;
#pragma unroll
                for (int r4 = 0; r4 < kRB; r4 += 4) {
                    const float4 s4 = lds_f32x4(sc + 4u * r4);
                    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const int r = r4 + rr;
#pragma unroll
                        for (int j = 0; j < BPL; ++j) {
                            const uint32_t b = (cw[sl][r] >> (8 * j)) & 0xFFu;
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                const float v = lds_f32(tl + 4u * (m * BPL + j) * kTableWords + b * 128u);
                                acc[m][r] = fmaf(v, sv[rr], acc[m][r]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (!lane_on) {
#pragma unroll
                    for (int r = 0; r < kRB; ++r) acc[m][r] = 0.f;
                }
                const float tot = transpose_reduce<kRB>(acc[m]);
                if (lane < kRB && r0 + lane < nrows) {
                    const int r = r0 + lane;
                    if (p.P == 1) {  // single pass: straight to the owner rank (no block barrier)
                        const int q = r / p.PER;
                        float* dst = cluster.map_shared_rank(red, q);
                        dst[(crank * MT + m) * p.PER + (r - q * p.PER)] = tot;
                    } else {
                        float* dst = acc_s + m * p.RP + r;
                        *dst = (pass == 0) ? tot : *dst + tot;
                    }
                }
            }
        };

        uint32_t cwA[NS][kRB], cwB[NS][kRB];
        // Code bytes do not depend on earlier kernels: request this warp's first
        // two batches before waiting for the activations.
        if (warp < nbatch) load_batch(warp, cwA);
        if (warp + kLutWarps < nbatch) load_batch(warp + kLutWarps, cwB);

        // decoded scales of this pass: ssc[gl][r]
        for (int r = threadIdx.x; r < p.RP; r += kLutThreads) {
            const uint16_t* sp = a.scales + (row0 + min(r, nrows - 1)) * a.ng + gg0;
            uint32_t sv[8];
#pragma unroll
            for (int gl = 0; gl < 8; ++gl) sv[gl] = gl < ngl ? __ldg(sp + gl) : 0u;
#pragma unroll
            for (int gl = 0; gl < 8; ++gl)
                if (gl < ngl) ssc[gl * p.RP + r] = r < nrows ? decoded_scale(sv[gl]) : 0.f;
        }
        if (pass == 0) {
            // Pull this CTA's code lines toward L2 before waiting for the activations.
            const int64_t span = (int64_t)ngl * B;  // bytes of one row in this pass
            const int nlines = (int)((span + 127) / 128) + 1;
            const int npf = min(nrows, 4096);
            for (int i = threadIdx.x; i < npf * nlines; i += kLutThreads) {
                const int r = i / nlines, l = i - r * nlines;
                const int64_t off = (int64_t)gg0 * B + (int64_t)l * 128;
                if (off < (int64_t)gg0 * B + span)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.codes + (row0 + r) * a.row_bytes + off));
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
        }

        // tables: work item = (slice, token, chunk position j, part d4 or NaN tail)
        const int items = NS * MT * BPL * 4;
        for (int it = warp; it < items; it += kLutWarps) {
            const int part = it & 3, j = (it >> 2) % BPL, m = ((it >> 2) / BPL) % MT;
            const int sl = (it >> 2) / (BPL * MT);
            float* tab = table + (size_t)((sl * MT + m) * BPL + j) * kTableWords;
            if (lane_on) build_part<B>(a, tab, sl, m, j, gg0, part);
        }
        __syncthreads();
        if (pass == 0) cluster_wait();  // every CTA of the cluster is running: partial rows may be pushed

        int bt = warp;
        while (bt < nbatch) {
            const int b1 = bt + kLutWarps;
            run_batch(bt, cwA);  // cwB (batch b1) is already in flight
            if (b1 >= nbatch) break;
            const int b2 = b1 + kLutWarps;
            if (b2 < nbatch) load_batch(b2, cwA);
            run_batch(b1, cwB);
            const int b3 = b2 + kLutWarps;
            if (b3 < nbatch) load_batch(b3, cwB);
            bt = b2;
        }
    }

    // Cluster reduction: every rank pushes its partial rows into the owner
    // rank's buffer (rows [q*PER, (q+1)*PER) belong to rank q), one cluster
    // barrier, then each owner adds the CS partials in rank order.
    if (p.P > 1) {
        __syncthreads();
        for (int i = threadIdx.x; i < nrows * MT; i += kLutThreads) {
            const int m = i / nrows, r = i - m * nrows;
            const int q = r / p.PER;
            float* dst = cluster.map_shared_rank(red, q);
            dst[(crank * MT + m) * p.PER + (r - q * p.PER)] = acc_s[m * p.RP + r];
        }
    }
    cluster.sync();
    const int rlo = crank * p.PER, rhi = min(nrows, rlo + p.PER);
    uint32_t err_acc = 0;
    for (int i = threadIdx.x; i < (rhi - rlo) * MT; i += kLutThreads) {
        const int m = i / (rhi - rlo), r = i - m * (rhi - rlo);
        float v = 0.f;
        for (int qr = 0; qr < p.CS; ++qr) v += red[(qr * MT + m) * p.PER + r];
        const int64_t n = row0 + rlo + r;
        if (v != v) err_acc |= scan_row_errors(a.codes + n * a.row_bytes, a.scales + n * a.ng, a.ng, a.G, B);
        const int64_t o = (int64_t)(a.m0 + m) * a.N + n;
        if (a.y_bf16) reinterpret_cast<__nv_bfloat16*>(a.Y)[o] = __float2bfloat16_rn(v);
        else reinterpret_cast<float*>(a.Y)[o] = v;
    }
    if (err_acc && a.d_err) atomicOr(a.d_err, err_acc);
}

// ---------------------------------------------------------------------------
// host side: plan + launch

static bool make_plan(int64_t N, int K, int G, int MT, int sm_count, size_t smem_limit, LutPlan* out) {
    const int B = bytes_per_group(G);
    const int ng = K / G;
    if ((B != 13 && B != 26) || ng % kGPS) return false;
    const int BPL = B / kLPG;
    const int S = ng / kGPS;
    const size_t table_per_slice = (size_t)MT * BPL * kTableWords * 4;
    const int ns_max = MT == 4 ? 1 : (MT == 2 ? 2 : 4);
    // Small matrices are latency-bound: keep two CTAs per SM.  Large ones
    // amortize bigger resident tables with one 512-thread CTA per SM.
    const bool big = (double)N * K > 16.0 * 1024 * 1024;
    const size_t smem_cap = big ? smem_limit : (size_t)112 * 1024;
    double best_cost = -1;
    LutPlan best{};
    for (int cs = 1; cs <= 8; ++cs) {
        if (S % cs) continue;
        const int per_cta = S / cs;
        for (int ns = 1; ns <= per_cta && ns <= ns_max; ++ns) {
            if (per_cta % ns || ns == 3) continue;
            const size_t tbytes = table_per_slice * ns;
            if (tbytes > (big ? (size_t)160 * 1024 : (size_t)96 * 1024)) continue;
            int rb = sm_count / cs;
            if (rb < 1) rb = 1;
            int64_t R = (N + rb - 1) / rb;
            if (R > 8192 || R * (int64_t)ng * B >= (int64_t(1) << 31)) continue;
            rb = (int)((N + R - 1) / R);
            const int64_t RP = (R + 31) / 32 * 32;
            const int64_t PER = (R + cs - 1) / cs;
            const size_t off_scale = tbytes;
            const size_t off_acc = off_scale + (size_t)ns * kGPS * RP * 4;
            const size_t off_red = off_acc + (size_t)MT * RP * 4;
            const size_t smem = off_red + (size_t)cs * MT * PER * 4;
            // two CTAs per SM, so a dependent launch's CTAs can start beside this one's
            if (smem > smem_cap) continue;
            // estimated cycles per CTA: table writes (one wavefront per 26 entries),
            // lookups (~1/20 cycle per byte per row), row reductions, cluster overhead
            const int passes = per_cta / ns;
            const double build = (double)passes * ns * MT * BPL * 256.0 * 1.2;
            const double look = (double)R * per_cta * kGPS * B * MT * 0.05;
            const double reduce = (double)R * passes * MT * 1.5;
            const double cost = build + look + reduce + 200.0 * cs;
            if (best_cost < 0 || cost < best_cost) {
                best_cost = cost;
                best.S = S;
                best.CS = cs;
                best.NS = ns;
                best.P = passes;
                best.R = (int)R;
                best.RP = (int)RP;
                best.RB = rb;
                best.MT = MT;
                best.PER = (int)PER;
                best.smem = smem;
                best.off_scale = off_scale;
                best.off_acc = off_acc;
                best.off_red = off_red;
            }
        }
    }
    if (best_cost < 0) return false;
    best.THREADS = big ? 512 : 256;
    *out = best;
    return true;
}

template <int B, int MT, int NS, int T>
static cudaError_t launch_lut(const LutArgs& a, cudaStream_t stream) {
    auto kern = gemv_lut_kernel<B, MT, NS, T>;
    static SmemAttr smem_attr;
    if (cudaError_t e = smem_attr.ensure(kern, (int)a.p.smem)) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.p.RB * a.p.CS));
    cfg.blockDim = dim3(T);
    cfg.dynamicSmemBytes = a.p.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.p.CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int B, int T>
static cudaError_t launch_lut_sel(const LutArgs& a, cudaStream_t stream) {
    const int ns = a.p.NS;
    switch (a.p.MT) {
        case 4: return launch_lut<B, 4, 1, T>(a, stream);
        case 2: return ns == 1 ? launch_lut<B, 2, 1, T>(a, stream) : launch_lut<B, 2, 2, T>(a, stream);
        default:
            return ns == 1 ? launch_lut<B, 1, 1, T>(a, stream)
                           : (ns == 2 ? launch_lut<B, 1, 2, T>(a, stream) : launch_lut<B, 1, 4, T>(a, stream));
    }
}

// Returns cudaErrorNotSupported when the shape is not covered (the caller
// then uses the row kernel).
cudaError_t launch_gemv_lut(const uint16_t* X, int64_t M, const uint8_t* codes, const uint16_t* scales,
                            int64_t N, int64_t K, int G, void* Y, int y_bf16, uint32_t* d_err,
                            cudaStream_t stream, int sm_count, size_t smem_limit) {
    if (M < 1 || M > 4 || M == 3 || K > (1 << 30) || N > (int64_t(1) << 40)) return cudaErrorNotSupported;
    const int MT = (int)M;
    LutArgs a{};
    if (!make_plan(N, (int)K, G, MT, sm_count, smem_limit, &a.p)) return cudaErrorNotSupported;
    const int B = bytes_per_group(G);
    if (B == 26 && (reinterpret_cast<uintptr_t>(codes) & 1)) return cudaErrorNotSupported;
    static const bool debug = getenv("TQ_DEBUG_PLAN") != nullptr;
    if (debug)
        fprintf(stderr, "tq gemv_lut N=%lld K=%lld G=%d M=%lld: S=%d CS=%d NS=%d P=%d R=%d RB=%d T=%d smem=%zu\n",
                (long long)N, (long long)K, G, (long long)M, a.p.S, a.p.CS, a.p.NS, a.p.P, a.p.R, a.p.RB,
                a.p.THREADS, a.p.smem);
    a.X = X;
    a.M = (int)M;
    a.m0 = 0;
    a.codes = codes;
    a.scales = scales;
    a.N = N;
    a.K = (int)K;
    a.G = G;
    a.ng = (int)(K / G);
    a.row_bytes = (int64_t)a.ng * B;
    a.Y = Y;
    a.y_bf16 = y_bf16;
    a.d_err = d_err;
    if (a.p.THREADS == 512) return B == 26 ? launch_lut_sel<26, 512>(a, stream) : launch_lut_sel<13, 512>(a, stream);
    return B == 26 ? launch_lut_sel<26, 256>(a, stream) : launch_lut_sel<13, 256>(a, stream);
}

}  // namespace tq
