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
// the mixed-precision FMA runs at 19 T/s, so the multiply-adds would saturate the
// SM.  Here each code costs ~0.7 integer instructions, and the multiply-adds go to
// the tensor cores through mma.sync m16n8k16 straight from registers (no shared
// memory round trip), which also makes M = 2..8 free: the MMA's n8 side is the batch.
//
//   * Codes become fp16 with a single AND: masking a word with 0x000F000F leaves two
//     fp16 SUBNORMALS q * 2^-24 (codes 0 and 4 of the word), 0x00F000F0 leaves
//     16 q * 2^-24 (codes 1 and 5); the word shifted right by 8 gives codes 2/6 and
//     3/7.  Products with x are exact in the fp32 accumulator.  The "x1" codes and
//     the "x16" codes go to two accumulators (D1, D16).
//   * The k order inside an MMA is free as long as A and B agree: lane (g, t) feeds
//     the k-slots of its quad with codes of its own word, and X is staged in shared
//     memory permuted the same way, so no shuffles or byte permutes are needed.
//   * The 4 lanes of a quad cover 32*WT consecutive codes (WT = 1, 2, 4 words each
//     for G = 32, 64, >= 128), which always lie inside one group, so after each
//     k-step the group's scale and zero point are applied once in fp32:
//       y += scale16 * (2^24 (D1 + D16/16) - z * sum_k x).
//   * Persistent CTAs: each stages X once and then walks row groups of 16 output
//     channels (rg = blockIdx.x, blockIdx.x + gridDim.x, ...).  Its 8 warps split K;
//     each warp keeps kGemvDepth k-steps of loads in flight across row-group
//     boundaries (a ring in registers), so the next row group streams in while the
//     current one is multiplied.  Per row group the 8 partial sums are added in a
//     fixed order (deterministic) through a double-buffered shared-memory slot.
//   * Programmatic dependent launch: weight loads are issued before
//     griddepcontrol.wait, so they overlap the previous kernel's tail; only X (the
//     previous layer's output in a model) is read after it.
#pragma once

#include "common.cuh"

namespace awq {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = 8;
constexpr int kGemvRows = 16;      // output channels per CTA (MMA M)
constexpr int kGemvDepth = 4;      // k-steps of loads in flight per warp

__host__ __device__ constexpr int gemv_words_per_thread(int G) { return G >= 128 ? 4 : G / 32; }

struct GemvSmem {
    // X permuted: [m][kstep][j][t] uint4, row pitch padded by 64 B; then xsum [m][kstep] fp32;
    // then partials [2 slots][warp][16 rows][8 m] fp32.
    static __host__ __device__ inline size_t x_pitch(int K) { return (size_t)K * 2 + 64; }
    static __host__ __device__ inline size_t xsum_off(int M, int K) { return (size_t)M * x_pitch(K); }
    static __host__ __device__ inline size_t part_off(int M, int K, int nsteps) {
        return (xsum_off(M, K) + (size_t)M * nsteps * 4 + 15) & ~(size_t)15;
    }
    static __host__ __device__ inline size_t bytes(int M, int K, int nsteps) {
        return part_off(M, K, nsteps) + (size_t)2 * kGemvWarps * kGemvRows * 8 * 4;
    }
};

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One k-step of loads in flight.  Everything is kept exactly as loaded: using a
// loaded value (even to pack or shift it) would stall the thread on the load.
template <int WT>
struct GemvStep {
    uint32_t wa[WT], wb[WT];   // code words of rows g and g+8
    uint32_t sa, sb;           // scale16 bits of rows g and g+8
    uint32_t za, zb;           // packed zero words of rows g and g+8
};

template <int WT>
__device__ __forceinline__ void load_words(const uint32_t* p, uint32_t (&w)[WT]) {
    if constexpr (WT == 4) {
        uint4 v;
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "l"(p));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (WT == 2) {
        uint2 v;
        asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
        w[0] = v.x; w[1] = v.y;
    } else {
        asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(w[0]) : "l"(p));
    }
}

template <int WT>
__global__ void __launch_bounds__(kGemvThreads, 2)
gemv_mma_kernel(const uint16_t* __restrict__ X, int M, const uint32_t* __restrict__ qweight,
                const uint16_t* __restrict__ scales, const uint32_t* __restrict__ qzeros, int N, int K, int G,
                int zero_point, uint16_t* __restrict__ Y) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int kStepCodes = 32 * WT;
    const int nsteps = K / kStepCodes;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int kw = K >> 3;
    const int ng = K / G;
    const int nzw = (ng + 7) >> 3;
    const bool zp = zero_point != 0;

    // The units of this warp are (row group, k-step) pairs: row groups
    // blockIdx.x + r * gridDim.x (r = 0 .. my_rg-1), k-steps s_begin .. s_begin+per-1 of
    // each.  k-steps at or beyond nsteps are empty, so every warp has the same unit
    // count and the per-row-group barrier below is uniform.  Cursors advance by one
    // unit at a time (no divisions in the loop).
    const int per = (nsteps + kGemvWarps - 1) / kGemvWarps;
    const int s_begin = warp * per;
    const int n_rg = (N + kGemvRows - 1) / kGemvRows;
    const int my_rg = blockIdx.x < n_rg ? (n_rg - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int U = my_rg * per;
    const int lg = 31 - __clz(G);            // G is a power of two

    // load cursor
    int l_rg = blockIdx.x, l_i = 0;
    auto load_next = [&](GemvStep<WT>& st) {
        const int s = s_begin + l_i;
        const int ra = l_rg * kGemvRows + g;
        const bool va = ra < N && s < nsteps, vb = ra + 8 < N && s < nsteps;
        const uint32_t* qa = qweight + (size_t)ra * kw + (s * 4 * WT + t * WT);
        const int grp = (s * kStepCodes) >> lg;
        if (va) {
            load_words<WT>(qa, st.wa);
        } else {
#pragma unroll
            for (int j = 0; j < WT; ++j) st.wa[j] = 0;
        }
        if (vb) {
            load_words<WT>(qa + 8 * (size_t)kw, st.wb);
        } else {
#pragma unroll
            for (int j = 0; j < WT; ++j) st.wb[j] = 0;
        }
        const uint16_t* sp = scales + (size_t)ra * ng + grp;
        st.sa = va ? __ldg(sp) : 0u;
        st.sb = vb ? __ldg(sp + 8 * (size_t)ng) : 0u;
        if (zp) {
            const uint32_t* zpp = qzeros + (size_t)ra * nzw + (grp >> 3);
            st.za = va ? __ldg(zpp) : 0u;
            st.zb = vb ? __ldg(zpp + 8 * (size_t)nzw) : 0u;
        } else {
            st.za = st.zb = 0x88888888u;   // implicit zero 8 in every nibble
        }
        if (++l_i == per) {
            l_i = 0;
            l_rg += gridDim.x;
        }
    };

    // 1. weights first (they do not depend on the previous kernel)
    GemvStep<WT> buf[kGemvDepth];
#pragma unroll
    for (int i = 0; i < kGemvDepth; ++i)
        if (i < U) load_next(buf[i]);

    // 2. wait for the producer of X, then stage it (permuted) and its per-step sums
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
                // x0..x7 -> (x0,x4) (x2,x6) (x1,x5) (x3,x7): the k-slots of the two MMAs of one word
                uint4 p;
                p.x = __byte_perm(v[i].x, v[i].z, 0x5410);
                p.y = __byte_perm(v[i].y, v[i].w, 0x5410);
                p.z = __byte_perm(v[i].x, v[i].z, 0x7632);
                p.w = __byte_perm(v[i].y, v[i].w, 0x7632);
                const int s = word / (4 * WT);
                const int r = word - s * 4 * WT;
                const int tt = r / WT, j = r - tt * WT;
                *reinterpret_cast<uint4*>(smem + m * pitch + ((size_t)(s * WT + j) * 4 + tt) * 16) = p;
            }
        }
    }
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
    const bool bm = g < M;   // lane supplies B column g
    const uint8_t* xrow = smem + g * pitch + t * 16;
    const int m0 = 2 * t, m1 = 2 * t + 1;
    const float* xs0 = xsum + m0 * nsteps;
    const float* xs1 = xsum + m1 * nsteps;
    float y[4] = {0.f, 0.f, 0.f, 0.f};
    int c_rg = blockIdx.x, c_i = 0, c_r = 0;   // consume cursor
    for (int u0 = 0; u0 < U; u0 += kGemvDepth) {
#pragma unroll
        for (int i = 0; i < kGemvDepth; ++i) {
            if (u0 + i >= U) break;
            const int s = s_begin + c_i;
            if (s < nsteps) {
                GemvStep<WT>& st = buf[i];
                float d1[4] = {0.f, 0.f, 0.f, 0.f}, d16[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < WT; ++j) {
                    uint4 b = make_uint4(0, 0, 0, 0);
                    if (bm) b = *reinterpret_cast<const uint4*>(xrow + (size_t)(s * WT + j) * 64);
                    const uint32_t wa = st.wa[j], wb = st.wb[j];
                    const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
                    mma_16816(d1, wa & 0x000F000Fu, wb & 0x000F000Fu, wa8 & 0x000F000Fu, wb8 & 0x000F000Fu, b.x, b.y);
                    mma_16816(d16, wa & 0x00F000F0u, wb & 0x00F000F0u, wa8 & 0x00F000F0u, wb8 & 0x00F000F0u, b.z,
                              b.w);
                }
                // fold this k-step's group scale and zero point (fp32); the 4-bit zero
                // becomes a float through the 2^23 magic number
                const float sa = h2f((uint16_t)st.sa), sb = h2f((uint16_t)st.sb);
                const int zsh = 4 * (((s * kStepCodes) >> lg) & 7);
                const float za = __uint_as_float(0x4B000000u | ((st.za >> zsh) & 15u)) - 8388608.0f;
                const float zb = __uint_as_float(0x4B000000u | ((st.zb >> zsh) & 15u)) - 8388608.0f;
                const float x0 = m0 < M ? xs0[s] : 0.f;
                const float x1 = m1 < M ? xs1[s] : 0.f;
                y[0] = fmaf(sa, fmaf(fmaf(d16[0], 0.0625f, d1[0]), 16777216.0f, -za * x0), y[0]);
                y[1] = fmaf(sa, fmaf(fmaf(d16[1], 0.0625f, d1[1]), 16777216.0f, -za * x1), y[1]);
                y[2] = fmaf(sb, fmaf(fmaf(d16[2], 0.0625f, d1[2]), 16777216.0f, -zb * x0), y[2]);
                y[3] = fmaf(sb, fmaf(fmaf(d16[3], 0.0625f, d1[3]), 16777216.0f, -zb * x1), y[3]);
            }
            if (u0 + i + kGemvDepth < U) load_next(buf[i]);
            if (++c_i == per) {
                // end of a row group: combine the 8 warps' partial sums in a fixed order
                float* slot = part + (c_r & 1) * (kGemvWarps * kGemvRows * 8);
                float* pw = slot + warp * kGemvRows * 8;
                pw[g * 8 + 2 * t] = y[0];
                pw[g * 8 + 2 * t + 1] = y[1];
                pw[(g + 8) * 8 + 2 * t] = y[2];
                pw[(g + 8) * 8 + 2 * t + 1] = y[3];
                y[0] = y[1] = y[2] = y[3] = 0.f;
                __syncthreads();
                if (threadIdx.x < kGemvRows * 8) {
                    const int r = threadIdx.x >> 3, m = threadIdx.x & 7;
                    float acc = 0.f;
#pragma unroll
                    for (int w = 0; w < kGemvWarps; ++w) acc += slot[w * kGemvRows * 8 + threadIdx.x];
                    const int n = c_rg * kGemvRows + r;
                    if (m < M && n < N) Y[(size_t)m * N + n] = f2h_rn(acc);
                }
                c_i = 0;
                c_rg += gridDim.x;
                ++c_r;
            }
        }
    }
}

}  // namespace awq
