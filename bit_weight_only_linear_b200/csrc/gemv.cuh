// Fused dequantising GEMV (decode, M <= 8): Y = X . deq(W)^T.
//
// Source: "Optimization Awq" (skillsdirectory.com), kernel backends (GEMV: batch size
// 1, single-token generation); "AI-Research-SKILLs AWQ advanced usage guide"
// (lshu.cn), WQLinear kernels.  Result as the header defines:
// y[m][n] = sum_k x[m][k] (q[n][k] - z[n][g]) scale16[n][g], exact products, fp32 sums.
//
// Why this shape (measured on B200): at M = 1 the kernel must turn 0.5 B of codes
// into one multiply-add at ~12.8 T codes/s to keep up with HBM.  On the CUDA cores
// the cheapest exact form (mask + fma.rn.f32.f16) costs ~2 issue slots per code and
// the mixed-precision FMA runs at 19 T/s, so the multiply-adds would saturate the SM.
// Here each code costs ~0.6 integer instructions, and the multiply-adds go to the
// tensor cores through mma.sync m16n8k16 straight from registers (no shared-memory
// round trip), which also makes M = 2..8 free: the MMA's n8 side is the batch.
//
//   * Codes become fp16 with a single AND: masking a word with 0x000F000F leaves two
//     fp16 SUBNORMALS q * 2^-24 (codes 0 and 4 of the word), 0x00F000F0 leaves
//     16 q * 2^-24 (codes 1 and 5); the word shifted right by 8 gives codes 2/6 and
//     3/7.  Products with x are exact in the fp32 accumulator.  The "x1" codes and
//     the "x16" codes go to two accumulators (D1, D16).
//   * The k order inside an MMA is free as long as A and B agree: lane (g, t) feeds
//     the k-slots of its quad with codes of its own word.  The packed order puts codes
//     k, k+1 at the same nibble of a word's two halves, so each mask leaves an adjacent
//     pair: the x1 MMA takes codes (0,1) and (4,5) of the word, the x16 MMA (2,3) and
//     (6,7).  One 16-byte load per lane holds x0..x7 of the word, staged as
//     (x0 x1, x4 x5, x2 x3, x6 x7) so that each MMA's B operand is a register pair
//     as loaded.
//   * X is staged with its 16-byte chunks reordered within each k-step to [j][t]: the
//     4 lanes of a quad then read 64 contiguous bytes, and with a row pitch of 64 mod
//     128 bytes the two rows of a quarter-warp fill all 32 banks (in natural order the
//     lanes t and t+2 would hit the same banks when WT = 4).
//   * The 4 lanes of a quad cover one k-step of 32*WT consecutive codes (WT = 1, 2, 4
//     words each for G = 32, 64, >= 128), which always lies inside one group, so after
//     each k-step the group's scale and zero point are applied once in fp32:
//       y += (scale16 * 2^24) (D1 + D16/16) - (scale16 * z) sum_k x.
//   * A unit is UK k-steps (8 words per row per lane).  Loads are never predicated:
//     rows past N are read from row N-1 and dropped at the store, k-steps past the
//     end are read from the last one with their scale forced to 0.
//   * Persistent CTAs stage X once, then walk row-group iterations.  KS warps split
//     the K of one 16-row group (KS = 1..8, chosen so that each warp has >= 4 units);
//     the CTA's 8 warps work on 8/KS row groups at a time.  Each warp keeps kGemvDepth
//     units of loads in flight across iterations (a ring in registers; loaded values
//     are stored untouched, since using a value stalls on its load).  Per iteration
//     the KS partial sums of a row are added in a fixed order (deterministic).
//   * Programmatic dependent launch: weight loads are issued before
//     griddepcontrol.wait, so they overlap the previous kernel's tail; only X (the
//     previous layer's output in a model) is read after it.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace awq {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 16;      // output channels per row group (MMA M)
constexpr int kGemvDepth = 2;      // units of loads in flight per warp
constexpr int kGemvUnitWords = 8;  // code words per row per lane per unit

__host__ __device__ constexpr int gemv_words_per_thread(int G) { return G >= 128 ? 4 : G / 32; }

struct GemvSmem {
    // X as [m][kstep][j][t] uint4, row pitch padded by 64 B; then xsum [m][kstep] fp32;
    // then partials [2 slots][8 warps][16 rows][8 m] fp32; then a 64-byte zero row.
    static __host__ __device__ inline size_t x_pitch(int K) { return (size_t)K * 2 + 64; }
    static __host__ __device__ inline size_t xsum_off(int M, int K) { return (size_t)M * x_pitch(K); }
    static __host__ __device__ inline size_t part_off(int M, int K, int nsteps) {
        return (xsum_off(M, K) + (size_t)M * nsteps * 4 + 15) & ~(size_t)15;
    }
    static __host__ __device__ inline size_t zero_off(int M, int K, int nsteps) {
        return part_off(M, K, nsteps) + (size_t)2 * kGemvWarps * kGemvRows * 8 * 4;
    }
    static __host__ __device__ inline size_t bytes(int M, int K, int nsteps) { return zero_off(M, K, nsteps) + 64; }
};

// K-split of one row group over KS warps: split further while a warp keeps at
// least 4 units, or (small N) while there are fewer row-group iterations than
// resident CTAs and a warp keeps at least one unit.
__host__ __device__ inline int gemv_ks(int units_per_row_group, int row_groups, int slots) {
    int ks = 1;
    while (ks < kGemvWarps &&
           (units_per_row_group >= 8 * ks ||
            (units_per_row_group >= 2 * ks && row_groups * ks / kGemvWarps < slots)))
        ks <<= 1;
    return ks;
}

// The MMA wrappers are not volatile: they are pure functions of their registers, and
// leaving the compiler free to interleave independent accumulation chains hides the
// MMA latency.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A * B (accumulator starts from zero).
__device__ __forceinline__ void mma_16816_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                uint32_t b0, uint32_t b1) {
    const float z = 0.0f;
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

template <int WT>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t* w) {
    if constexpr (WT == 4) {
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "l"(p));
    } else if constexpr (WT == 2) {
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "l"(p));
    } else {
        asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(w[0]) : "l"(p));
    }
}

// One unit of loads in flight (UK k-steps of rows g and g+8), kept exactly as loaded.
// A unit covers 256 consecutive codes starting at a multiple of 256, i.e. 256/G whole
// groups (or part of one when G = 256) starting at a multiple of 256/G, so all of
// its zero points sit in one packed zero word (8 groups per word).
template <int UK>
struct GemvUnit {
    uint32_t wa[kGemvUnitWords], wb[kGemvUnitWords];   // code words of rows g and g+8
    uint32_t sa[UK], sb[UK];                           // scale16 bits per k-step
    uint32_t za, zb;                                   // packed zero word of the unit
};

template <int WT, bool ONE>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv_mma_kernel(const uint16_t* __restrict__ X, int M, const uint32_t* __restrict__ qweight,
                const uint16_t* __restrict__ scales, const uint32_t* __restrict__ qzeros, int N, int K, int G,
                int zero_point, int ks_arg, uint16_t* __restrict__ Y) {
    constexpr int UK = kGemvUnitWords / WT;   // k-steps per unit
    constexpr int kStepCodes = 32 * WT;
    extern __shared__ __align__(16) uint8_t smem[];
    const int nsteps = K / kStepCodes;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int kw = K >> 3;
    const int ng = K / G;
    const int nzw = (ng + 7) >> 3;
    const bool zp = zero_point != 0;
    const int lg = 31 - __clz(G);            // G is a power of two

    // K split: KS warps per row group, RPI = 8/KS row groups per CTA iteration.
    const int units = (nsteps + UK - 1) / UK;                 // units per row group
    const int KS = ks_arg;
    const int RPI = kGemvWarps / KS;
    const int sub = warp / KS;                                // which row group of the iteration
    const int kpart = warp - sub * KS;                        // which K part
    const int per = (units + KS - 1) / KS;                    // units per warp per row group
    const int u_begin = kpart * per;
    const int n_rg = (N + kGemvRows - 1) / kGemvRows;
    const int n_it = (n_rg + RPI - 1) / RPI;                  // row-group iterations in total
    const int my_it = blockIdx.x < n_it ? (n_it - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int U = my_it * per;                                // units of this warp

    // load cursor: iteration l_it (row group l_it * RPI + sub), unit u_begin + l_i
    int l_it = blockIdx.x, l_i = 0;
    auto load_next = [&](GemvUnit<UK>& st) {
        const int rg = l_it * RPI + sub;
        const int ra = min(rg * kGemvRows + g, N - 1);
        const int rb = min(rg * kGemvRows + g + 8, N - 1);
        const uint32_t* qa = qweight + (size_t)ra * kw + t * WT;
        const uint32_t* qb = qweight + (size_t)rb * kw + t * WT;
        const int s0 = (u_begin + l_i) * UK;
        const uint16_t* spa = scales + (size_t)ra * ng;
        const uint16_t* spb = scales + (size_t)rb * ng;
#pragma unroll
        for (int k = 0; k < UK; ++k) {
            const int s = min(s0 + k, nsteps - 1);
            load_words<WT>(qa + s * 4 * WT, st.wa + k * WT);
            load_words<WT>(qb + s * 4 * WT, st.wb + k * WT);
            const int grp = (s * kStepCodes) >> lg;
            st.sa[k] = __ldg(spa + grp);
            st.sb[k] = __ldg(spb + grp);
        }
        if (zp) {
            const int grp0 = (min(s0, nsteps - 1) * kStepCodes) >> lg;
            st.za = __ldg(qzeros + (size_t)ra * nzw + (grp0 >> 3));
            st.zb = __ldg(qzeros + (size_t)rb * nzw + (grp0 >> 3));
        } else {
            st.za = st.zb = 0x88888888u;   // implicit zero 8 in every nibble
        }
        if (++l_i == per) {
            l_i = 0;
            l_it += gridDim.x;
        }
    };

    // 1. weights first (they do not depend on the previous kernel)
    GemvUnit<UK> buf[kGemvDepth];
#pragma unroll
    for (int i = 0; i < kGemvDepth; ++i)
        if (i < U) load_next(buf[i]);

    // 2. wait for the producer of X, then stage it (chunks reordered) and its per-step sums
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const size_t pitch = GemvSmem::x_pitch(K);
    float* xsum = reinterpret_cast<float*>(smem + GemvSmem::xsum_off(M, K));
    float* part = reinterpret_cast<float*>(smem + GemvSmem::part_off(M, K, nsteps));
    // all global loads of a thread are issued before any of its shared-memory stores
    constexpr int kStageUnroll = 4;
    for (int u0 = threadIdx.x; u0 < M * kw; u0 += kGemvThreads * kStageUnroll) {
        uint4 v[kStageUnroll];
#pragma unroll
        for (int i = 0; i < kStageUnroll; ++i) {
            const int u = u0 + i * kGemvThreads;
            if (u < M * kw) {
                const int m = u / kw;
                v[i] = __ldg(reinterpret_cast<const uint4*>(X + (size_t)m * K + (u - m * kw) * 8));
            }
        }
#pragma unroll
        for (int i = 0; i < kStageUnroll; ++i) {
            const int u = u0 + i * kGemvThreads;
            if (u < M * kw) {
                const int m = u / kw;
                const int word = u - m * kw;
                const int s = word / (4 * WT);
                const int r = word - s * 4 * WT;
                const int tt = r / WT, j = r - tt * WT;
                *reinterpret_cast<uint4*>(smem + m * pitch + ((size_t)(s * WT + j) * 4 + tt) * 16) =
                    make_uint4(v[i].x, v[i].z, v[i].y, v[i].w);
            }
        }
    }
    if (threadIdx.x < 16)
        reinterpret_cast<uint32_t*>(smem + GemvSmem::zero_off(M, K, nsteps))[threadIdx.x] = 0u;
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // per-(m, k-step) sums of x, from shared memory, in a fixed order
    for (int u = threadIdx.x; u < M * nsteps; u += kGemvThreads) {
        const int m = u / nsteps;
        const int s = u - m * nsteps;
        const uint4* xr = reinterpret_cast<const uint4*>(smem + m * pitch) + (size_t)s * WT * 4;
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < 4 * WT; ++i) {
            const uint4 v = xr[i];
            const uint16_t* h = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc += h2f(h[e]);
        }
        xsum[u] = acc;
    }
    __syncthreads();

    // 3. stream the units; D fragment: y[0] = (row g, col 2t), y[1] = (g, 2t+1),
    //    y[2] = (g+8, 2t), y[3] = (g+8, 2t+1)
    // lanes whose B column is past M read the zero row staged after X
    // lane (g, t) reads x0..x7 of word t*WT + j of each k-step, staged at chunk j*4 + t
    const uint8_t* xrow = (g < M ? smem + g * pitch : smem + GemvSmem::zero_off(M, K, nsteps)) + t * 16;
    const size_t xstep = g < M ? 64 : 0;
    const int m0 = 2 * t, m1 = 2 * t + 1;
    const float* xs0 = xsum + (m0 < M ? m0 : 0) * nsteps;
    const float* xs1 = xsum + (m1 < M ? m1 : 0) * nsteps;
    const float xm0 = m0 < M ? 1.0f : 0.0f, xm1 = m1 < M ? 1.0f : 0.0f;
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    int c_it = blockIdx.x, c_i = 0, c_r = 0;   // consume cursor
    for (int u0 = 0; u0 < U; u0 += kGemvDepth) {
#pragma unroll
        for (int i = 0; i < kGemvDepth; ++i) {
            if (u0 + i >= U) break;
            GemvUnit<UK>& st = buf[i];
            const int s0 = (u_begin + c_i) * UK;
#pragma unroll
            for (int k = 0; k < UK; ++k) {
                const int s = s0 + k;
                const int sc = min(s, nsteps - 1);
                float d1[4], d16[4];
#pragma unroll
                for (int j = 0; j < WT; ++j) {
                    const uint4 b = *reinterpret_cast<const uint4*>(xrow + (size_t)(sc * WT + j) * xstep);
                    const uint32_t wa = st.wa[k * WT + j], wb = st.wb[k * WT + j];
                    const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
                    if (j == 0) {
                        mma_16816_first(d1, wa & 0x000F000Fu, wb & 0x000F000Fu, wa8 & 0x000F000Fu,
                                        wb8 & 0x000F000Fu, b.x, b.y);
                        mma_16816_first(d16, wa & 0x00F000F0u, wb & 0x00F000F0u, wa8 & 0x00F000F0u,
                                        wb8 & 0x00F000F0u, b.z, b.w);
                    } else {
                        mma_16816(d1, wa & 0x000F000Fu, wb & 0x000F000Fu, wa8 & 0x000F000Fu, wb8 & 0x000F000Fu,
                                  b.x, b.y);
                        mma_16816(d16, wa & 0x00F000F0u, wb & 0x00F000F0u, wa8 & 0x00F000F0u, wb8 & 0x00F000F0u,
                                  b.z, b.w);
                    }
                }
                // fold the k-step's group scale and zero point; k-steps past the end get scale 0
                const float on = s < nsteps ? 1.0f : 0.0f;
                const float sa = h2f((uint16_t)st.sa[k]) * on, sb = h2f((uint16_t)st.sb[k]) * on;
                const int zsh = 4 * (((sc * kStepCodes) >> lg) & 7);
                // the 4-bit zero becomes a float through the 2^23 magic number
                const float za = __uint_as_float(0x4B000000u | ((st.za >> zsh) & 15u)) - 8388608.0f;
                const float zb = __uint_as_float(0x4B000000u | ((st.zb >> zsh) & 15u)) - 8388608.0f;
                const float sa24 = sa * 16777216.0f, sb24 = sb * 16777216.0f;
                const float x0 = xs0[sc] * xm0;
                y[0] = fmaf(sa24, fmaf(d16[0], 0.0625f, d1[0]), fmaf(-sa * za, x0, y[0]));
                y[2] = fmaf(sb24, fmaf(d16[2], 0.0625f, d1[2]), fmaf(-sb * zb, x0, y[2]));
                if (!ONE) {
                    const float x1 = xs1[sc] * xm1;
                    y[1] = fmaf(sa24, fmaf(d16[1], 0.0625f, d1[1]), fmaf(-sa * za, x1, y[1]));
                    y[3] = fmaf(sb24, fmaf(d16[3], 0.0625f, d1[3]), fmaf(-sb * zb, x1, y[3]));
                }
            }
            if (u0 + i + kGemvDepth < U) load_next(buf[i]);
            if (++c_i == per) {
                // end of an iteration: combine the KS partial sums of each row in a fixed order
                float* slot = part + (c_r & 1) * (kGemvWarps * kGemvRows * 8);
                float* pw = slot + warp * kGemvRows * 8;
                pw[g * 8 + 2 * t] = y[0];
                pw[g * 8 + 2 * t + 1] = y[1];
                pw[(g + 8) * 8 + 2 * t] = y[2];
                pw[(g + 8) * 8 + 2 * t + 1] = y[3];
                y[0] = y[1] = y[2] = y[3] = 0.f;
                __syncthreads();
                for (int o = threadIdx.x; o < RPI * kGemvRows * 8; o += kGemvThreads) {
                    const int sb2 = o / (kGemvRows * 8);
                    const int e = o - sb2 * (kGemvRows * 8);
                    const int r = e >> 3, m = e & 7;
                    float acc = 0.f;
                    for (int w = 0; w < KS; ++w) acc += slot[(sb2 * KS + w) * kGemvRows * 8 + e];
                    const int n = (c_it * RPI + sb2) * kGemvRows + r;
                    if (m < M && n < N) Y[(size_t)m * N + n] = f2h_rn(acc);
                }
                c_i = 0;
                c_it += gridDim.x;
                ++c_r;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// TMA-staged GEMV for N % 16 == 0 (every real layer): the same arithmetic as
// gemv_mma_kernel with a different data path.
//   * Weights reach shared memory through one 3-D tensor TMA copy per stage
//     (16 rows x 2048 codes = 16 KB) issued by a producer warp into a ring of S
//     stages.  The 3-D view {16 words, rows, 128-code blocks} lands a stage as
//     [block][row][64 B], so the two rows a quarter-warp reads are adjacent and the
//     shared loads are conflict-free (row-major stages gave 8-way conflicts).
//     Measured on B200: 16 per-row bulk copies per stage cap the copy rate near
//     2 TB/s; one tensor copy per stage does not.  The producer waits for a free
//     stage and, once, for the X copy to have been requested (see kTmaStagesBeforeX).
//   * Scales and zero words of a row group arrive through two bulk copies into a
//     ring of PR raw parameter slots, all issued by the producer before its first
//     weight stage when they fit.  A converter warp turns the groups of each
//     stage into fp32 pairs (scale16 * 2^24, scale16 * zero) in a small buffer that
//     belongs to the stage: a stage is full when both its TMA bytes and the
//     converter's arrival are in, and both refill it after the consumers release
//     it.  Per-stage buffers keep the footprint of long rows small enough for two
//     CTAs per SM.
//   * The 8 consumer warps run only the decode, the MMAs and the fold, each taking
//     1/8 of a stage's k-steps; a reducer warp adds their partial sums in a fixed
//     order.  Every wait is bounded.
// ---------------------------------------------------------------------------

// Warp roles: producer, converter and reducer are warps 0-2, the consumers warps 3-10.
constexpr int kTmaConsumers = 8;                            // consumer warps
constexpr int kTmaProducerWarp = 0;                         // weight TMA copies
constexpr int kTmaConverterWarp = 1;                        // scale/zero copies -> fp32 pairs
constexpr int kTmaReducerWarp = 2;                          // partial sums -> Y
constexpr int kTmaFirstConsumer = 3;                        // consumers: warps 3 .. 10
constexpr int kTmaThreads = (kTmaConsumers + 3) * 32;
constexpr int kTmaMinStages = 3, kTmaMaxStages = 6;
constexpr int kTmaMaxParamSlots = 8;
// Weight stages a CTA requests before X has been requested.  X is the first thing the
// consumers need and arrives only after the previous kernel has completed; a full ring
// of weight requests issued ahead of it (up to 24 MB over the GPU) was measured to delay
// its arrival, while two stages keep the early prefetch.
constexpr int kTmaStagesBeforeX = 2;
constexpr int kTmaKC = 2048;                                // codes per row per stage
constexpr int kTmaBlkBytes = kGemvRows * 64;               // one 128-code block of 16 rows
constexpr int kTmaStageBytes = (kTmaKC / 128) * kTmaBlkBytes;

struct GemvTmaSmem {
    // K is padded to whole stages (Kp) in every shared-memory copy: X and its step sums
    // are zero past K and so are the converted parameters past the last group, so the
    // last, partial stage needs no validity checks.
    int K, M, S, PR, Kp, nstepsp, ng, nzw, gpc;
    __host__ __device__ GemvTmaSmem(int M_, int K_, int G, int S_, int PR_) : K(K_), M(M_), S(S_), PR(PR_) {
        Kp = (K + kTmaKC - 1) / kTmaKC * kTmaKC;
        nstepsp = Kp / (32 * gemv_words_per_thread(G));
        ng = K / G;
        nzw = (ng + 7) / 8;
        gpc = kTmaKC / G;
    }
    static __host__ __device__ size_t al16(size_t x) { return (x + 15) & ~(size_t)15; }
    __host__ __device__ size_t raw_scale_bytes() const { return (size_t)kGemvRows * ng * 2; }
    __host__ __device__ size_t raw_zero_bytes() const { return (size_t)kGemvRows * nzw * 4; }
    __host__ __device__ size_t raw_stride() const { return al16(raw_scale_bytes()) + al16(raw_zero_bytes()); }
    __host__ __device__ size_t cvt_stride() const { return (size_t)kGemvRows * gpc * 8; }
    __host__ __device__ size_t part_stride() const { return (size_t)kTmaConsumers * kGemvRows * M * 4; }
    __host__ __device__ size_t raw() const { return (size_t)S * kTmaStageBytes; }
    __host__ __device__ size_t cvt() const { return raw() + PR * raw_stride(); }
    __host__ __device__ size_t x() const { return al16(cvt() + S * cvt_stride()); }
    __host__ __device__ size_t xsum() const { return x() + (size_t)M * GemvSmem::x_pitch(Kp); }
    __host__ __device__ size_t part() const { return al16(xsum() + (size_t)M * nstepsp * 4); }
    __host__ __device__ size_t bars() const { return (part() + 2 * part_stride() + 7) & ~(size_t)7; }
    // full[S], empty[S], pfull[PR], rfull[2], rempty[2], xfull, xissued
    __host__ __device__ size_t bytes() const { return bars() + (2 * S + PR + 6) * 8; }
};

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(sm100::smem_u32(dst)), "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float ldsf(uint32_t a) { return __uint_as_float(lds32(a)); }

template <int WT>
__device__ __forceinline__ void lds_words(uint32_t a, uint32_t* w) {
    if constexpr (WT == 4) {
        const uint4 v = lds128(a);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (WT == 2) {
        const uint2 v = lds64(a);
        w[0] = v.x; w[1] = v.y;
    } else {
        w[0] = lds32(a);
    }
}

// G is a template parameter so that every group index is a shift.  S (stages) and
// PR (raw parameter slots) are chosen by the host from the shared-memory budget.
template <int G, bool ONE>
__global__ void __launch_bounds__(kTmaThreads, 2)
gemv_tma_kernel(const __grid_constant__ CUtensorMap tmap_q, const uint16_t* __restrict__ X, int M,
                const uint16_t* __restrict__ scales, const uint32_t* __restrict__ qzeros, int N, int K,
                int zero_point, uint16_t* __restrict__ Y, int S, int PR) {
    using namespace sm100;
    constexpr int WT = gemv_words_per_thread(G);
    constexpr int kStepCodes = 32 * WT;
    constexpr int kStepsPerStage = kTmaKC / kStepCodes;
    constexpr int Q = kStepsPerStage / kTmaConsumers;           // k-steps of a warp per stage
    constexpr int GPC = kTmaKC / G;                             // groups per stage
    extern __shared__ __align__(16) uint8_t smem[];
    const GemvTmaSmem L(M, K, G, S, PR);
    const int ng = L.ng, nzw = L.nzw, nstepsp = L.nstepsp;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool zp = zero_point != 0;
    const int n_rg = N / kGemvRows;
    const int my_rg = blockIdx.x < n_rg ? (n_rg - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int nchunks = L.Kp / kTmaKC;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars());   // weights + converted params in
    uint64_t* empty = full + S;                 // consumers done with a stage
    uint64_t* pfull = empty + S;                // raw parameters of a row group landed
    uint64_t* rfull = pfull + PR;               // partial sums of a row group written
    uint64_t* rempty = rfull + 2;               // reducer done with a partial-sum slot
    uint64_t* xfull = rempty + 2;               // X rows landed
    uint64_t* xissued = xfull + 1;              // X copy requested

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 2);             // producer (with its bytes) + converter
            mbar_init(&empty[i], kTmaConsumers);
        }
        for (int i = 0; i < PR; ++i) mbar_init(&pfull[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&rfull[i], kTmaConsumers);
            mbar_init(&rempty[i], 1);
        }
        mbar_init(xfull, 1);
        mbar_init(xissued, 1);
        mbar_fence_init();
        prefetch_tensormap(&tmap_q);
    }
    __syncthreads();

    // raw scales/zeros of row group j into slot j % PR (one thread)
    const uint32_t pbytes = (uint32_t)(L.raw_scale_bytes() + (zp ? L.raw_zero_bytes() : 0));
    auto issue_params = [&](int j) {
        const int p = j % PR;
        const int r0 = (blockIdx.x + j * gridDim.x) * kGemvRows;
        uint8_t* raw = smem + L.raw() + p * L.raw_stride();
        mbar_arrive_expect_tx(&pfull[p], pbytes);
        bulk_g2s(raw, scales + (size_t)r0 * ng, (uint32_t)L.raw_scale_bytes(), &pfull[p]);
        if (zp)
            bulk_g2s(raw + L.al16(L.raw_scale_bytes()), qzeros + (size_t)r0 * nzw, (uint32_t)L.raw_zero_bytes(),
                     &pfull[p]);
    };
    if (warp == kTmaProducerWarp) {
        // ---------------- producer: the first parameter copies, then the weight stream,
        // gated by free stages and, after kTmaStagesBeforeX stages, by the X copy having
        // been requested (parameters and X first so that they do not queue behind the
        // weights) ----------------
        if (lane == 0) {
            for (int j = 0; j < PR && j < my_rg; ++j) issue_params(j);
            bool ok = true;
            int stage = 0, st = 0;
            uint32_t ph = 0;                    // parity of the current use of slot st
            for (int rgi = 0; rgi < my_rg && ok; ++rgi) {
                const int r0 = (blockIdx.x + rgi * gridDim.x) * kGemvRows;
                for (int c = 0; c < nchunks; ++c) {
                    if (stage == kTmaStagesBeforeX && !(ok = mbar_wait(xissued, 0))) break;
                    if (stage >= S && !(ok = mbar_wait(&empty[st], ph ^ 1u))) break;
                    // box {16 words, 16 rows, 16 blocks}; blocks past K are filled with zeros
                    mbar_arrive_expect_tx(&full[st], kTmaStageBytes);
                    tma_load_3d(smem + (size_t)st * kTmaStageBytes, &tmap_q, &full[st], 0, r0, c * (kTmaKC / 128));
                    ++stage;
                    if (++st == S) { st = 0; ph ^= 1u; }
                }
            }
            // drain: copies in flight must land before the CTA exits
            for (int s2 = stage - 1; s2 >= 0 && s2 >= stage - S; --s2) mbar_wait(&full[s2 % S], (s2 / S) & 1);
        }
        return;
    }
    if (warp == kTmaConverterWarp) {
        // ---------------- converter: raw scales/zeros of a row group -> per-stage
        // (scale16 * 2^24, scale16 * zero) pairs; refills the raw slots ----------------
        int issued = my_rg < PR ? my_rg : PR;
        bool ok = true;
        int rgi = 0, stage = 0, st = 0;
        uint32_t ph = 0;
        // vector form: a lane takes 8 consecutive groups of one row (one 16-byte scale
        // load, one zero word, four 16-byte stores); needs 16-byte aligned scale rows
        const bool vec = (ng & 7) == 0;
        constexpr int OCT = GPC / 8;                          // octets of groups per row per stage
        constexpr int IPL = (kGemvRows * OCT + 31) / 32;      // octets per lane
        constexpr int EPL = kGemvRows * GPC / 32;             // (row, group) pairs per lane (scalar form)
        constexpr int EB = EPL < 8 ? EPL : 8;
        for (; rgi < my_rg && ok; ++rgi) {
            const int p = rgi % PR;
            if (!(ok = mbar_wait(&pfull[p], (rgi / PR) & 1))) break;
            const uint8_t* raw = smem + L.raw() + p * L.raw_stride();
            const uint16_t* rs = reinterpret_cast<const uint16_t*>(raw);
            const uint32_t* rz = reinterpret_cast<const uint32_t*>(raw + L.al16(L.raw_scale_bytes()));
            for (int c = 0; c < nchunks; ++c) {
                if (stage >= S && !(ok = mbar_wait(&empty[st], ph ^ 1u))) break;
                float2* cv = reinterpret_cast<float2*>(smem + L.cvt() + (size_t)st * L.cvt_stride());
                if (vec) {
#pragma unroll
                    for (int i = 0; i < IPL; ++i) {
                        const int it = lane + 32 * i;
                        if (it < kGemvRows * OCT) {
                            const int r = it / OCT, o = it % OCT;
                            const int g0 = c * GPC + 8 * o;
                            uint4 v = make_uint4(0u, 0u, 0u, 0u);   // groups past K contribute nothing
                            uint32_t zw = 0u;
                            if (g0 < ng) {
                                v = *reinterpret_cast<const uint4*>(rs + r * ng + g0);
                                if (zp) zw = rz[r * nzw + (g0 >> 3)];
                            }
                            const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
                            float4 out[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const float s0 = h2f((uint16_t)(hw[k] & 0xFFFFu)), s1 = h2f((uint16_t)(hw[k] >> 16));
                                const float z0 = zp ? (float)((zw >> (8 * k)) & 15u) : 8.0f;
                                const float z1 = zp ? (float)((zw >> (8 * k + 4)) & 15u) : 8.0f;
                                out[k] = make_float4(s0 * 16777216.0f, s0 * z0, s1 * 16777216.0f, s1 * z1);
                            }
                            float4* dst = reinterpret_cast<float4*>(cv + r * GPC + 8 * o);
#pragma unroll
                            for (int k = 0; k < 4; ++k) dst[k] = out[k];
                        }
                    }
                } else {
                    for (int i0 = 0; i0 < EPL; i0 += EB) {
                        float sc[EB];
                        uint32_t zw[EB];
#pragma unroll
                        for (int i = 0; i < EB; ++i) {
                            const int e = lane + 32 * (i0 + i);
                            const int r = e / GPC, grp = c * GPC + (e % GPC);
                            const bool live = grp < ng;   // groups past K contribute nothing
                            sc[i] = live ? h2f(rs[r * ng + grp]) : 0.0f;
                            zw[i] = (live && zp) ? rz[r * nzw + (grp >> 3)] : 0u;
                        }
#pragma unroll
                        for (int i = 0; i < EB; ++i) {
                            const int e = lane + 32 * (i0 + i);
                            const int grp = c * GPC + (e % GPC);
                            const float z = zp ? (float)((zw[i] >> (4 * (grp & 7))) & 15u) : 8.0f;
                            cv[e] = make_float2(sc[i] * 16777216.0f, sc[i] * z);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[st]);
                ++stage;
                if (++st == S) { st = 0; ph ^= 1u; }
            }
            if (!ok) break;
            // the whole warp has read raw slot p: refill it
            if (lane == 0 && rgi + PR < my_rg) issue_params(rgi + PR);
            if (rgi + PR < my_rg) ++issued;
        }
        // after a timeout, parameter copies still in flight must land before the CTA exits
        if (lane == 0)
            for (int j = issued - 1; j >= rgi && j >= issued - PR; --j) mbar_wait(&pfull[j % PR], (j / PR) & 1);
        return;
    }
    if (warp == kTmaReducerWarp) {
        // ---------------- reducer: add the 8 partial sums of each output in a fixed order ----------------
        const float* part = reinterpret_cast<const float*>(smem + L.part());
        for (int rgi = 0; rgi < my_rg; ++rgi) {
            const int b = rgi & 1;
            if (!mbar_wait(&rfull[b], (rgi >> 1) & 1)) break;
            const float* slot = part + b * (L.part_stride() / 4);
            const int n0 = (blockIdx.x + rgi * gridDim.x) * kGemvRows;
            for (int o = lane; o < kGemvRows * M; o += 32) {
                const int r = o / M, m = o - r * M;
                float acc = 0.f;
#pragma unroll
                for (int w = 0; w < kTmaConsumers; ++w) acc += slot[w * kGemvRows * M + o];
                Y[(size_t)m * N + n0 + r] = f2h_rn(acc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[b]);
        }
        return;
    }

    // ---------------- consumers: stage X (chunks reordered, zero past K) and its per-step sums ----------------
    const int cw = warp - kTmaFirstConsumer;          // consumer index 0..7
    const int ct = threadIdx.x - kTmaFirstConsumer * 32;
    // One bulk copy per X row lands the rows in natural order; each round then reads 256
    // 16-byte chunks (whole k-steps of one row), and after a barrier writes them back in
    // place in the [j][t] order the B fragments read, while the lanes of each k-step add
    // up its activations.
    const size_t pitch = GemvSmem::x_pitch(L.Kp);
    uint8_t* xs = smem + L.x();
    float* xsum = reinterpret_cast<float*>(smem + L.xsum());
    constexpr int kCons = kTmaConsumers * 32;
    if (ct == 0) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        mbar_arrive_expect_tx(xfull, (uint32_t)M * (uint32_t)K * 2u);
        for (int m = 0; m < M; ++m) bulk_g2s(xs + m * pitch, X + (size_t)m * K, (uint32_t)K * 2u, xfull);
        mbar_arrive(xissued);
    }
    bool ok = mbar_wait(xfull, 0);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    {
        constexpr int TPS = 4 * WT;                     // chunks (lanes) per k-step
        const int kwp = L.Kp >> 3;                      // chunks per padded row
        const int kwv = K >> 3;                         // chunks per row that hold data
        for (int u0 = 0; u0 < M * kwp; u0 += kCons) {   // kwp is a multiple of kCons
            const int u = u0 + ct;
            const int m = u0 / kwp;
            const int word = u - m * kwp;
            uint4* row = reinterpret_cast<uint4*>(xs + m * pitch);
            const uint4 v = word < kwv ? row[word] : make_uint4(0u, 0u, 0u, 0u);   // zero past K
            asm volatile("bar.sync 1, %0;" ::"n"(kCons) : "memory");
            const int s = word / TPS, r = word % TPS;
            const int tt = r / WT, j = r % WT;
            row[(s * WT + j) * 4 + tt] = make_uint4(v.x, v.z, v.y, v.w);
            const uint16_t* h = reinterpret_cast<const uint16_t*>(&v);
            float acc = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc += h2f(h[e]);
#pragma unroll
            for (int o = TPS / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (r == 0) xsum[m * nstepsp + s] = acc;
        }
        // (a round writes only the chunks it read, so rounds need no barrier between them)
        asm volatile("bar.sync 1, %0;" ::"n"(kCons) : "memory");
    }

    // ---------------- consumers: stream the stages ----------------
    // Every per-k-step shared address below is a per-stage base plus a compile-time
    // offset.  Lanes whose B column is past M read X row 0: their D columns are never
    // used, and a uniform stride keeps the offsets constant.
    constexpr int kStepsPerBlk = 4 / WT;             // k-steps per 128-code block
    constexpr int R = G >= kStepCodes ? G / kStepCodes : 1;   // k-steps per group
    const int g = lane >> 2, t = lane & 3;
    const uint32_t sbase = smem_u32(smem);
    // lane (g, t) reads x0..x7 of word t*WT + j of each k-step, staged at chunk j*4 + t
    const uint32_t xrow = smem_u32(xs + (g < M ? g : 0) * pitch) + t * 16 + (uint32_t)(cw * Q * WT * 64);
    const int m0 = 2 * t, m1 = 2 * t + 1;
    const uint32_t xs0 = smem_u32(xsum + (m0 < M ? m0 : 0) * nstepsp) + (uint32_t)(cw * Q * 4);
    const uint32_t xs1 = smem_u32(xsum + (m1 < M ? m1 : 0) * nstepsp) + (uint32_t)(cw * Q * 4);
    const float xm0 = m0 < M ? 1.0f : 0.0f, xm1 = m1 < M ? 1.0f : 0.0f;
    float* part = reinterpret_cast<float*>(smem + L.part());
    // weights: word w of row r in block b of a stage sits at b * kTmaBlkBytes + r * 64 + w * 4;
    // this warp's first k-step of a stage starts a block (cw * Q is a multiple of kStepsPerBlk)
    const uint32_t wrow = (uint32_t)((cw * Q / kStepsPerBlk) * kTmaBlkBytes + g * 64 + t * WT * 4);
    // converted parameters of a stage: [row][group of the stage] fp32 pairs
    const uint32_t prow = smem_u32(smem + L.cvt()) + (uint32_t)(g * GPC * 8 + ((cw * Q) / R) * 8);
    const uint32_t cstride = (uint32_t)L.cvt_stride();

    int st = 0;
    uint32_t ph = 0;
    for (int rgi = 0; rgi < my_rg; ++rgi) {
        float y[4] = {0.f, 0.f, 0.f, 0.f};
        for (int c = 0; c < nchunks; ++c) {
            ok = ok && mbar_wait(&full[st], ph);
            const uint32_t sb = sbase + (uint32_t)(st * kTmaStageBytes) + wrow;
            const uint32_t cva = prow + (uint32_t)st * cstride;
            const uint32_t xb = xrow + (uint32_t)(c * kStepsPerStage * WT * 64);
            const uint32_t x0b = xs0 + (uint32_t)(c * kStepsPerStage * 4);
            const uint32_t x1b = xs1 + (uint32_t)(c * kStepsPerStage * 4);
            // the warp's Q k-steps as straight-line code: fragment loads, then independent
            // MMA chains interleaved, then the folds
            uint32_t wa[Q][WT], wb[Q][WT];
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const uint32_t off = (uint32_t)((q / kStepsPerBlk) * kTmaBlkBytes + (q % kStepsPerBlk) * WT * 16);
                lds_words<WT>(sb + off, wa[q]);
                lds_words<WT>(sb + off + 8 * 64, wb[q]);
            }
            float d1[Q][4], d16[Q][4];
#pragma unroll
            for (int j = 0; j < WT; ++j) {
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    const uint4 b = lds128(xb + (uint32_t)((q * WT + j) * 64));
                    const uint32_t a = wa[q][j], bb = wb[q][j];
                    const uint32_t a8 = a >> 8, b8 = bb >> 8;
                    if (j == 0) {
                        mma_16816_first(d1[q], a & 0x000F000Fu, bb & 0x000F000Fu, a8 & 0x000F000Fu,
                                        b8 & 0x000F000Fu, b.x, b.y);
                        mma_16816_first(d16[q], a & 0x00F000F0u, bb & 0x00F000F0u, a8 & 0x00F000F0u,
                                        b8 & 0x00F000F0u, b.z, b.w);
                    } else {
                        mma_16816(d1[q], a & 0x000F000Fu, bb & 0x000F000Fu, a8 & 0x000F000Fu, b8 & 0x000F000Fu,
                                  b.x, b.y);
                        mma_16816(d16[q], a & 0x00F000F0u, bb & 0x00F000F0u, a8 & 0x00F000F0u,
                                  b8 & 0x00F000F0u, b.z, b.w);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                // fold: y += (scale16 2^24) (D1 + D16/16) - (scale16 z) sum_k x
                const uint32_t go = (uint32_t)((q / R) * 8);
                const uint2 pa = lds64(cva + go);
                const uint2 pbv = lds64(cva + go + 8 * GPC * 8);
                const float x0 = ldsf(x0b + (uint32_t)(q * 4)) * xm0;
                const float sa = __uint_as_float(pa.x), sza = __uint_as_float(pa.y);
                const float sb2 = __uint_as_float(pbv.x), szb = __uint_as_float(pbv.y);
                y[0] = fmaf(sa, fmaf(d16[q][0], 0.0625f, d1[q][0]), fmaf(-sza, x0, y[0]));
                y[2] = fmaf(sb2, fmaf(d16[q][2], 0.0625f, d1[q][2]), fmaf(-szb, x0, y[2]));
                if (!ONE) {
                    const float x1 = ldsf(x1b + (uint32_t)(q * 4)) * xm1;
                    y[1] = fmaf(sa, fmaf(d16[q][1], 0.0625f, d1[q][1]), fmaf(-sza, x1, y[1]));
                    y[3] = fmaf(sb2, fmaf(d16[q][3], 0.0625f, d1[q][3]), fmaf(-szb, x1, y[3]));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
            if (++st == S) { st = 0; ph ^= 1u; }
        }
        // hand the partial sums to the reducer warp (no CTA-wide barrier)
        const int b = rgi & 1;
        if (rgi >= 2) ok = ok && mbar_wait(&rempty[b], ((rgi >> 1) - 1) & 1);
        float* pw = part + b * (L.part_stride() / 4) + cw * kGemvRows * M;
        if (m0 < M) {
            pw[g * M + m0] = y[0];
            pw[(g + 8) * M + m0] = y[2];
        }
        if (m1 < M) {
            pw[g * M + m1] = y[1];
            pw[(g + 8) * M + m1] = y[3];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rfull[b]);
    }
}

}  // namespace awq
