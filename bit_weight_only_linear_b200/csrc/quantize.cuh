// Group quantise + pack, activation statistic, alpha -> s, and the activation fold.
//
// Source of the arithmetic: "AI-Research-SKILLs AWQ advanced usage guide"
// (lshu.cn), sections 算法原理 (scale s from activation statistics, W*s quantised,
// s^-1 folded into X) and 量化超参数调优 (group size; zero-point = offset for
// asymmetric ranges, off = symmetric), with the quantiser the library fixes:
// scale = (max-min)/15 or max|w|/7, zero = clamp(rint(-min/scale), 0, 15),
// q = clamp(rint(w/scale) + zero, 0, 15), all IEEE fp32, round-half-even.
#pragma once

#include "common.cuh"

namespace awq {

// Bit position of code j (0..7) in a qweight word: codes k, k+1 share a nibble position
// in the low and high 16-bit halves (nibbles 0, 4, 1, 5, 2, 6, 3, 7), so one mask of the
// word yields the adjacent pair (k, k+1) as the tensor-core fragments take it.
__host__ __device__ constexpr int code_shift(int j) { return 4 * ((j >> 1) + 4 * (j & 1)); }   // 0,16,4,20,8,24,12,28

constexpr int kQuantThreads = 256;                 // 8 elements per thread
constexpr int kQuantChunk = kQuantThreads * 8;     // 2048 input channels per block
constexpr float kScaleFloor = 1e-5f;

// The two fp32 products of the fp16 pairs in w and s (each exact: 11-bit x 11-bit
// significands fit in fp32), by the mixed-precision FMA with a -0 addend: no conversion
// instructions, and a zero keeps its sign like the plain fp32 product.
__device__ __forceinline__ void mul_f16x2_f32(uint32_t w, uint32_t s, float& lo, float& hi) {
    asm("{\n\t.reg .f16 wl, wh, sl, sh;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "mov.b32 {sl, sh}, %3;\n\t"
        "fma.rn.f32.f16 %0, wl, sl, 0f80000000;\n\t"
        "fma.rn.f32.f16 %1, wh, sh, 0f80000000;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(w), "r"(s));
}

// Round to the nearest integer, ties to even, for |x| < 2^22, by adding and removing
// 1.5 * 2^23 (two FP32 adds instead of a rounding instruction).  Larger |x| gives some
// value of magnitude >= 2^21, which callers either clamp or re-check.
__device__ __forceinline__ float rint_magic(float x) {
    return __fsub_rn(__fadd_rn(x, 12582912.0f), 12582912.0f);
}

struct GroupParams {
    float sc;     // fp32 value of the fp16 scale
    float rc;     // fl(1 / sc), correctly rounded
    float zero;   // integer-valued
    uint16_t sc16;
};

// rint(fl(ws / sc)) (IEEE fp32 division, then round half to even) with the division
// done only near a rounding boundary.  With rc = fl(1/sc) and t = fl(ws * rc), the
// standard error model gives |t - ws/sc| <= |ws/sc| (2^-24 + 2^-24 + 2^-48), and fl(ws/sc)
// is within |ws/sc| 2^-24 of ws/sc; so if t is farther than |t| 2^-21 from the nearest
// half-integer, ws/sc, t and fl(ws/sc) lie strictly on the same side of it (and fl(ws/sc)
// is no tie), and rint(t) = rint(fl(ws/sc)).  Otherwise the exact division decides.
__device__ __forceinline__ float rint_quotient(float ws, float sc, float rc) {
    const float t = __fmul_rn(ws, rc);
    const float half_dist = fabsf(__fsub_rn(__fsub_rn(t, floorf(t)), 0.5f));
    if (half_dist > fabsf(t) * 0x1p-21f) return rintf(t);
    return rintf(__fdiv_rn(ws, sc));
}

// Per-group scale/zero from the group's extreme values, as the header defines.
__device__ __forceinline__ GroupParams group_params(float mx, float mn, bool zero_point) {
    GroupParams p;
    if (zero_point) {
        float scale32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        scale32 = fmaxf(scale32, kScaleFloor);
        p.sc16 = f2h_rn(scale32);
        p.sc = h2f(p.sc16);
        p.rc = __frcp_rn(p.sc);
        p.zero = fminf(fmaxf(rint_quotient(-mn, p.sc, p.rc), 0.0f), 15.0f);
    } else {
        float amax = fmaxf(fabsf(mx), fabsf(mn));
        float scale32 = __fdiv_rn(amax, 7.0f);
        scale32 = fmaxf(scale32, kScaleFloor);
        p.sc16 = f2h_rn(scale32);
        p.sc = h2f(p.sc16);
        p.rc = __frcp_rn(p.sc);
        p.zero = 8.0f;
    }
    return p;
}

// Code of one scaled weight.
__device__ __forceinline__ uint32_t quant_code(float ws, const GroupParams& p, bool zero_point) {
    float r = rint_quotient(ws, p.sc, p.rc);
    if (zero_point) return (uint32_t)fminf(fmaxf(r + p.zero, 0.0f), 15.0f);
    return (uint32_t)(fminf(fmaxf(r, -8.0f), 7.0f) + 8.0f);
}

// Butterfly max/min over the `seg` consecutive lanes (power of two) that hold a group.
__device__ __forceinline__ void seg_minmax(float& mx, float& mn, int seg) {
    for (int off = seg >> 1; off > 0; off >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    }
}

// One block per (4 rows, 2048-channel chunk); thread t owns channels [8t, 8t+8) of the
// chunk in each of the 4 rows and writes one qweight word per row.  The 4 rows' loads
// are issued together, so their latency overlaps the quantisation of the rows before.
// A group of G channels spans G/8 lanes of one warp, so its min/max is a shuffle
// butterfly; the chunk holds whole zero words (2048/G groups, a multiple of 8), packed
// through shared memory.
constexpr int kQuantRows = 4;

// Codes of 8 scaled weights of one group, packed into one word, from the group's
// reciprocal scale rc = fl(1/sc) and its clamp bounds in the biased domain below.
//  * Rounding: t = fl(q + 1.5 * 2^23) with q = fl(ws * rc) holds rint(q) (ties to even)
//    as an integer in its significand while |q| < 2^22, and r = t - 1.5 * 2^23 and
//    e = q - r are exact.
//  * Exactness: q is within |ws/sc| (2^-23 + 2^-48) of ws/sc and fl(ws/sc) within
//    |ws/sc| 2^-24, so for |ws/sc| <= 33 the two differ by less than 2^-17.  Then
//    |e| < 1/2 - 2^-17 puts fl(ws/sc) strictly inside r's rounding interval, so
//    rint(fl(ws/sc)) = r.  When |q| >= 32 the code is clamped to the same end of the
//    range for any rounding of the quotient, so the test may pass there too.  If any of
//    the 8 fails, all 8 take the IEEE division.
//  * Clamp and pack: the clamp to [lo, hi] happens on t, against the bounds
//    1.5 * 2^23 + lo and 1.5 * 2^23 + hi.  Near 1.5 * 2^23 the bit pattern of a float is
//    linear in its integer value, so bits(t) - (bits(1.5 * 2^23) - off) is the code,
//    with off = zero, or 8 when symmetric.  The 8 codes are summed at their nibbles from
//    the raw bits (mod 2^32), and the 8 copies of that bias are removed at once:
//    bias * 0x11111111.  The codes lie in 0..15 at distinct nibbles, so no carry crosses
//    a nibble.
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;   // its bit pattern

__device__ __forceinline__ uint32_t pack_codes8(const float (&ws)[8], float rc, uint32_t sz, bool zp) {
    float t[8];
    bool good = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float q = __fmul_rn(ws[i], rc);
        t[i] = __fadd_rn(q, kMagic);
        const float e = __fsub_rn(q, __fsub_rn(t[i], kMagic));
        good = good && (fabsf(e) < 0.5f - 0x1p-17f);
    }
    if (!good) {
        const float sc = h2f((uint16_t)(sz & 0xFFFFu));
#pragma unroll
        for (int i = 0; i < 8; ++i) t[i] = __fadd_rn(rintf(__fdiv_rn(ws[i], sc)), kMagic);
    }
    const uint32_t zero = sz >> 16;
    const uint32_t off = zp ? zero : 8u;
    const float tlo = __uint_as_float(kMagicBits - off);           // 1.5 * 2^23 + lo
    const float thi = __uint_as_float(kMagicBits + 15u - off);     // 1.5 * 2^23 + hi
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc += __float_as_uint(fminf(fmaxf(t[i], tlo), thi)) << code_shift(i);
    return acc - (kMagicBits - off) * 0x11111111u;
}

// One block per (4 rows, 2048-channel chunk); thread t owns channels [8t, 8t+8) of the
// chunk in each of the 4 rows and writes one qweight word per row.  The 4 rows are loaded
// together; a group's min/max is a shuffle butterfly over its G/8 lanes.  The scale and
// zero point of each (row, group) are then computed once per warp: a warp holds
// 4 x 256/G <= 32 such pairs, lane p computes pair p and the lanes fetch their groups'
// parameters back by shuffles.  The chunk holds whole zero words (2048/G groups, a
// multiple of 8), packed through shared memory.
// G is a template parameter: every group index, lane count and shuffle loop is then a
// compile-time shift or an unrolled sequence (with a run-time G they were integer
// divisions and loops, a large share of the instructions per element).
template <int G>
__global__ void __launch_bounds__(kQuantThreads, 4)
quantize_pack_kernel(const uint16_t* __restrict__ W, const uint16_t* __restrict__ s, int N, int K,
                     int zero_point, uint32_t* __restrict__ qweight,
                     uint16_t* __restrict__ scales, uint32_t* __restrict__ qzeros) {
    __shared__ uint8_t zbuf[kQuantRows][kQuantChunk / 32];
    const int nchunks = ceil_div(K, kQuantChunk);
    const int row0 = (blockIdx.x / nchunks) * kQuantRows;
    const int chunk = blockIdx.x % nchunks;
    const int k0 = chunk * kQuantChunk + threadIdx.x * 8;
    const int lane = threadIdx.x & 31;
    const bool active = k0 < K;
    const bool zp = zero_point != 0;
    const int ng = K / G;

    uint4 wv[kQuantRows];
#pragma unroll
    for (int r = 0; r < kQuantRows; ++r) {
        wv[r] = make_uint4(0u, 0u, 0u, 0u);
        if (active && row0 + r < N) wv[r] = *reinterpret_cast<const uint4*>(W + (size_t)(row0 + r) * K + k0);
    }
    uint4 sv = make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);   // s = 1
    if (s != nullptr && active) sv = *reinterpret_cast<const uint4*>(s + k0);
    // ws = W s (exact), kept for both passes; the group extremes of each row
    float ws[kQuantRows][8];
    float gmx[kQuantRows], gmn[kQuantRows];
#pragma unroll
    for (int r = 0; r < kQuantRows; ++r) {
        mul_f16x2_f32(wv[r].x, sv.x, ws[r][0], ws[r][1]);
        mul_f16x2_f32(wv[r].y, sv.y, ws[r][2], ws[r][3]);
        mul_f16x2_f32(wv[r].z, sv.z, ws[r][4], ws[r][5]);
        mul_f16x2_f32(wv[r].w, sv.w, ws[r][6], ws[r][7]);
        float mx = fmaxf(ws[r][0], ws[r][1]), mn = fminf(ws[r][0], ws[r][1]);
#pragma unroll
        for (int i = 2; i < 8; i += 2) {
            mx = fmax3(mx, ws[r][i], ws[r][i + 1]);
            mn = fmin3(mn, ws[r][i], ws[r][i + 1]);
        }
#pragma unroll
        for (int off = (G >> 3) >> 1; off > 0; off >>= 1) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        }
        gmx[r] = mx;
        gmn[r] = mn;
    }
    // the parameters of pair p = (row p / gpw, group p % gpw of the warp), once per pair
    constexpr int L = G >> 3;             // lanes per group
    constexpr int gpw = 32 / L;           // groups per warp and row
    const int pr = lane / gpw, pg = lane - pr * gpw;
    float pmx = 0.0f, pmn = 0.0f;
#pragma unroll
    for (int r = 0; r < kQuantRows; ++r) {
        const float a = __shfl_sync(0xffffffffu, gmx[r], pg * L);
        const float b = __shfl_sync(0xffffffffu, gmn[r], pg * L);
        if (pr == r) pmx = a, pmn = b;
    }
    const GroupParams P = group_params(pmx, pmn, zp);
    const uint32_t psz = (uint32_t)P.sc16 | ((uint32_t)P.zero << 16);
#pragma unroll
    for (int r = 0; r < kQuantRows; ++r) {
        const int src = r * gpw + lane / L;
        const float rc = __shfl_sync(0xffffffffu, P.rc, src);
        const uint32_t sz = __shfl_sync(0xffffffffu, psz, src);
        const int row = row0 + r;                       // uniform over the block
        if (active && row < N) {
            qweight[(size_t)row * (K >> 3) + (k0 >> 3)] = pack_codes8(ws[r], rc, sz, zp);
            if ((k0 % G) == 0) {
                const int g = k0 / G;
                scales[(size_t)row * ng + g] = (uint16_t)(sz & 0xFFFFu);
                zbuf[r][(threadIdx.x * 8) / G] = (uint8_t)(sz >> 16);
            }
        }
    }
    if (!zp) return;
    __syncthreads();
    const int groups_here = kQuantChunk / G;          // multiple of 8
    const int g_base = chunk * groups_here;
    const int words = groups_here / 8;
    for (int t = threadIdx.x; t < kQuantRows * words; t += kQuantThreads) {
        const int r = t / words, zw = t - r * words;
        const int row = row0 + r;
        if (row < N && g_base + zw * 8 < ng) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) {
                const int g = g_base + zw * 8 + i;
                if (g < ng) word |= (uint32_t)zbuf[r][zw * 8 + i] << (4 * i);
            }
            qzeros[(size_t)row * ceil_div(ng, 8) + (g_base >> 3) + zw] = word;
        }
    }
}

// A kernel with no work, enqueued right after a kernel that writes packed weights.  The
// GEMV is launched as a programmatic dependent and streams its weights before it waits
// for the previous kernel on the stream, so that previous kernel must not be the one
// that wrote them; this one is launched with an ordinary stream dependency, so it
// starts only after the writer has completed and its stores are visible.
__global__ void stream_order_kernel() {}

// Column sums of |X| in fp64.  Every partial sum is an exact fp64 number (fp16
// values are multiples of 2^-24 and the sums stay far below 2^29), so the atomic
// accumulation is exact and order-independent.  Block: 128 threads x 8 columns;
// grid.y splits the rows.
__global__ void __launch_bounds__(128)
abs_colsum_kernel(const uint16_t* __restrict__ X, int M, int K, double* __restrict__ colsum) {
    const int c0 = (blockIdx.x * 128 + threadIdx.x) * 8;
    if (c0 >= K) return;
    const int rows_per = ceil_div(M, gridDim.y);
    const int r0 = blockIdx.y * rows_per;
    const int r1 = min(M, r0 + rows_per);
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    for (int r = r0; r < r1; ++r) {
        const uint4 v = *reinterpret_cast<const uint4*>(X + (size_t)r * K + c0);
        const uint16_t* h = reinterpret_cast<const uint16_t*>(&v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += (double)fabsf(h2f(h[i]));
    }
    if (r1 > r0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) atomicAdd(colsum + c0 + i, acc[i]);
    }
}

// s[a][k] = fp16(max(pow(colsum[k]/M, a/n_grid), 2^-14)) for every alpha of the grid.
__global__ void scales_for_alphas_kernel(const double* __restrict__ colsum, int M, int K,
                                         int n_grid, uint16_t* __restrict__ s_all) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    const int a = blockIdx.y;
    if (k >= K) return;
    const double m = __ddiv_rn(colsum[k], (double)M);
    const double alpha = __ddiv_rn((double)a, (double)n_grid);
    double p = pow(m, alpha);
    p = fmax(p, 6.103515625e-05);   // 2^-14
    s_all[(size_t)a * K + k] = d2h_rn(p);
}

// X_out = fp16(fp32(X) / fp32(s)), 8 elements per thread, grid-stride.
__global__ void fold_inverse_scale_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ s,
                                          int M, int K, uint16_t* __restrict__ Xo) {
    const size_t total8 = (size_t)M * K / 8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total8;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i * 8;
        const int k = (int)(e % K);
        const uint4 xv = *reinterpret_cast<const uint4*>(X + e);
        const uint4 sv = *reinterpret_cast<const uint4*>(s + k);
        const uint16_t* xh = reinterpret_cast<const uint16_t*>(&xv);
        const uint16_t* sh = reinterpret_cast<const uint16_t*>(&sv);
        uint4 ov;
        uint16_t* oh = reinterpret_cast<uint16_t*>(&ov);
#pragma unroll
        for (int j = 0; j < 8; ++j) oh[j] = f2h_rn(__fdiv_rn(h2f(xh[j]), h2f(sh[j])));
        *reinterpret_cast<uint4*>(Xo + e) = ov;
    }
}

}  // namespace awq
