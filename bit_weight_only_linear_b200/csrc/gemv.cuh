// Fused dequantising GEMV (decode, M <= 8): Y = X . deq(W)^T.
//
// Source: "Optimization Awq" (skillsdirectory.com), section on kernel backends
// (GEMV: batch size 1, single-token generation) and "AI-Research-SKILLs AWQ
// advanced usage guide" (lshu.cn), section on the WQLinear kernels.  The result
// is the one the header defines: y[m][n] = sum_k x[m][k] (q[n][k] - z) scale16.
//
// Design (HBM-bound: 0.5 B of codes per multiply-add at M = 1):
//   * A warp owns R output rows at a time and streams them in 1024-channel
//     chunks: lane l reads one 16-byte word group (32 consecutive codes) per row
//     per chunk, so a row's 2 KiB (K = 4096) is read as fully coalesced 512-byte
//     warp transactions.  Loads for the next chunk are issued before the current
//     chunk is computed (register double buffering).
//   * X is staged once per block in shared memory, permuted so that the 16-byte
//     pieces lane l needs are bank-conflict free, together with per-lane-chunk sums
//     of x used to fold the zero point out of the inner loop:
//         sum_k x (q - z) = sum_k x q - z sum_k x.
//   * Nibbles are turned into fp16 without any conversion instruction: masking a
//     word with 0x000F000F leaves two fp16 SUBNORMALS q*2^-24 (codes 0 and 4 of
//     the word), masking with 0x00F000F0 leaves 16 q * 2^-24 (codes 1 and 5); the
//     word shifted by 8 gives codes 2/6 and 3/7.  Each is multiplied by x with the
//     sm_100 mixed-precision fma.rn.f32.f16 (exact product, fp32 accumulate), so
//     the inner loop costs 13 instructions per 8 codes and is exact up to fp32
//     accumulation.  The 2^24 and the scale are applied once per (row, chunk).
#pragma once

#include "common.cuh"

namespace awq {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvChunk = 1024;   // input channels per warp step (32 lanes x 32)

// acc_even += sum over the word's even codes of x*q*2^-24, acc_odd += sum over odd codes of x*16q*2^-24.
__device__ __forceinline__ void dot_word(uint32_t w, uint4 x, float& ae, float& ao) {
    const uint32_t lo = w & 0x000F000Fu;
    const uint32_t hi = w & 0x00F000F0u;
    const uint32_t w8 = w >> 8;
    const uint32_t lo2 = w8 & 0x000F000Fu;
    const uint32_t hi2 = w8 & 0x00F000F0u;
    asm("{\n\t"
        ".reg .f16 l0, l1, h0, h1, m0, m1, g0, g1, x0, x1, x2, x3, x4, x5, x6, x7;\n\t"
        "mov.b32 {l0, l1}, %2;\n\t"
        "mov.b32 {h0, h1}, %3;\n\t"
        "mov.b32 {m0, m1}, %4;\n\t"
        "mov.b32 {g0, g1}, %5;\n\t"
        "mov.b32 {x0, x1}, %6;\n\t"
        "mov.b32 {x2, x3}, %7;\n\t"
        "mov.b32 {x4, x5}, %8;\n\t"
        "mov.b32 {x6, x7}, %9;\n\t"
        "fma.rn.f32.f16 %0, l0, x0, %0;\n\t"
        "fma.rn.f32.f16 %0, l1, x4, %0;\n\t"
        "fma.rn.f32.f16 %0, m0, x2, %0;\n\t"
        "fma.rn.f32.f16 %0, m1, x6, %0;\n\t"
        "fma.rn.f32.f16 %1, h0, x1, %1;\n\t"
        "fma.rn.f32.f16 %1, h1, x5, %1;\n\t"
        "fma.rn.f32.f16 %1, g0, x3, %1;\n\t"
        "fma.rn.f32.f16 %1, g1, x7, %1;\n\t"
        "}"
        : "+f"(ae), "+f"(ao)
        : "r"(lo), "r"(hi), "r"(lo2), "r"(hi2), "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w));
}

__device__ __forceinline__ uint4 ldg_stream(const uint32_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__host__ __device__ constexpr int gemv_rows_per_warp(int mt) { return mt <= 2 ? 4 : (mt <= 4 ? 2 : 1); }

// Shared memory bytes for a given padded batch MT and K.
__host__ __device__ inline size_t gemv_smem_bytes(int mt, int K) {
    const int nc = ceil_div(K, kGemvChunk);
    return (size_t)mt * nc * (4 * 32 * 16 + 32 * 4);
}

struct GemvChunkLoad {
    uint4 w;
    float sc;
    float z;
};

template <int MT, int R>
__global__ void __launch_bounds__(kGemvThreads)
gemv_kernel(const uint16_t* __restrict__ X, int M, const uint32_t* __restrict__ qweight,
            const uint16_t* __restrict__ scales, const uint32_t* __restrict__ qzeros, int N, int K,
            int G, int zero_point, uint16_t* __restrict__ Y) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int nc = ceil_div(K, kGemvChunk);
    uint4* xs = reinterpret_cast<uint4*>(smem);                                    // [MT][nc][4][32]
    float* csum = reinterpret_cast<float*>(smem + (size_t)MT * nc * 4 * 32 * 16);  // [MT][nc][32]

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int kw = K >> 3;                 // qweight words per row
    const int ng = K / G;
    const int nzw = ceil_div(ng, 8);
    const bool zp = zero_point != 0;
    const int row_groups = ceil_div(N, R);
    const int gwarp = blockIdx.x * kGemvWarps + warp;
    const int nwarps = gridDim.x * kGemvWarps;

    auto load_chunk = [&](int n0, int c, GemvChunkLoad (&out)[R]) {
        const int k = c * kGemvChunk + lane * 32;
        const int g = k / G;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int n = n0 + r;
            if (n < N && k < K) {
                out[r].w = ldg_stream(qweight + (size_t)n * kw + (k >> 3));
                out[r].sc = h2f(__ldg(scales + (size_t)n * ng + g));
                out[r].z = zp ? (float)((__ldg(qzeros + (size_t)n * nzw + (g >> 3)) >> (4 * (g & 7))) & 15u)
                              : 8.0f;
            } else {
                out[r].w = make_uint4(0, 0, 0, 0);
                out[r].sc = 0.0f;
                out[r].z = 0.0f;
            }
        }
    };

    // Start the first weight loads before staging X, so DRAM latency overlaps it.
    GemvChunkLoad cur[R], nxt[R];
    int rg = gwarp;
    if (rg < row_groups) load_chunk(rg * R, 0, cur);

    // Stage X (zero padded to MT rows and nc*1024 channels) in the permuted layout.
    const int units = MT * nc * 128;   // 16-byte units
    for (int u = threadIdx.x; u < units; u += kGemvThreads) {
        const int m = u / (nc * 128);
        const int rem = u - m * nc * 128;
        const int k = rem * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M && k < K) v = *reinterpret_cast<const uint4*>(X + (size_t)m * K + k);
        const int c = k >> 10, l = (k >> 5) & 31, j = (k >> 3) & 3;
        xs[((m * nc + c) * 4 + j) * 32 + l] = v;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < MT * nc * 32; t += kGemvThreads) {
        const int l = t & 31;
        const int mc = t >> 5;
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 v = xs[(mc * 4 + j) * 32 + l];
            const uint16_t* h = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc += h2f(h[e]);
        }
        csum[t] = acc;
    }
    __syncthreads();

    for (; rg < row_groups; rg += nwarps) {
        const int n0 = rg * R;
        float y[R][MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) y[r][m] = 0.0f;

        for (int c = 0; c < nc; ++c) {
            if (c + 1 < nc) {
                load_chunk(n0, c + 1, nxt);
            } else if (rg + nwarps < row_groups) {
                load_chunk((rg + nwarps) * R, 0, nxt);
            }
            float ae[R][MT], ao[R][MT];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) ae[r][m] = ao[r][m] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 xv[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) xv[m] = xs[((m * nc + c) * 4 + j) * 32 + lane];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint32_t w = j == 0 ? cur[r].w.x : j == 1 ? cur[r].w.y : j == 2 ? cur[r].w.z : cur[r].w.w;
#pragma unroll
                    for (int m = 0; m < MT; ++m) dot_word(w, xv[m], ae[r][m], ao[r][m]);
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float cx = csum[(m * nc + c) * 32 + lane];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float t = fmaf(ao[r][m], 0.0625f, ae[r][m]);
                    const float u = fmaf(t, 16777216.0f, -cur[r].z * cx);
                    y[r][m] = fmaf(cur[r].sc, u, y[r][m]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) cur[r] = nxt[r];
        }

#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float v = y[r][m];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                y[r][m] = v;
            }
        if (lane == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int n = n0 + r;
                if (n < N) {
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m < M) Y[(size_t)m * N + n] = f2h_rn(y[r][m]);
                }
            }
        }
    }
}

}  // namespace awq
