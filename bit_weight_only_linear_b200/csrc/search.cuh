// Activation-aware scale search on the sm_100a tensor cores, with the pseudo-quantisation
// fused into the producer of the loss GEMM.
//
// Source: "AI-Research-SKILLs AWQ advanced usage guide" (lshu.cn), section 算法原理:
// choose the per-input-channel scale s that minimises L(s) = || Q(W s)(s^-1 X) - W X ||,
// with s derived from the activation distribution; the search space is
// s = mean|X|^alpha over a grid of alpha.  Per alpha (the quantiser's steps in IEEE
// fp32 as in awq_quantize_pack, the loss in fp64):
//   m_k    = mean_t |X[t][k]|                       (exact: fp64 sums of fp16 values)
//   s_k    = fp16(max(pow(m_k, alpha), 2^-14))
//   dW     = (Q(W s) - W s) / s  = Q(W s)/s - W
//   loss   = mean_{t,n} (sum_k X[t][k] dW[n][k])^2
//
// One CTA takes one alpha, 128 output channels and up to 512 calibration tokens.  Its
// sixteen producer warps read W straight from memory and build dW tile by tile: the
// group's min/max (a shuffle over the four lanes that hold a row's 64-channel block),
// scale and zero point, the codes, and dW, which they scale by a power of two 2^e (one
// per alpha, from a bound on |dW|) and split into two fp16 terms hi + lo (a 22-bit
// significand).  The two terms go into 128-byte-swizzled shared-memory tiles that are
// the A operand of tcgen05.mma; X arrives by TMA as the B operand (two tiles of 256
// tokens), and E = X hi^T + X lo^T accumulates in fp32 in tensor memory (two 256-column
// accumulators).  The epilogue undoes 2^e and sums E^2 in fp64.  Neither dW nor E ever
// reaches global memory; tile partial sums are added in a fixed order, so the loss is
// deterministic.
//
// The exponent.  For a group g with scaled-weight magnitudes up to a = max|W s|,
// |Q(Ws) - Ws| <= |q - z| scale16 + a <= 3.001 a + 1.51e-4 (scale16 <= 2a/15 with zero
// point, a/7 without, floored at fp16(1e-5)), and a <= max|W|_g max s_g, so
// |dW| <= B = max_g (3.01 max|W|_g max s_g + 1.6e-4) / min s_g, with max|W|_g taken over
// all rows.  2^e puts B just below 2^15: hi stays finite in fp16 and every |dW| within
// 2^17 of the bound keeps all 22 bits.
#pragma once

#include "common.cuh"
#include "gemm_sm100.cuh"
#include "quantize.cuh"
#include "sm100.cuh"

namespace awq {

constexpr int kSearchMaxGrid = 64;     // n_grid upper bound
constexpr int kSearchRows = 128;       // output channels per CTA (MMA M)
constexpr int kSearchTokTile = 256;    // tokens per accumulator (MMA N)
constexpr int kSearchTokChunk = 512;   // tokens per CTA (two accumulators)
constexpr int kSearchXStages = 2;
constexpr int kSearchABufs = 2;
constexpr int kSearchProducerWarps = 16;
constexpr int kSearchThreads = 64 + kSearchProducerWarps * 32;   // TMA warp, MMA warp, producers

struct FusedSearchCfg {
    static constexpr int kXTileBytes = kSearchTokTile * 128;    // 256 tokens x 64 channels fp16
    static constexpr int kXStageBytes = 2 * kXTileBytes;
    static constexpr int kATileBytes = kSearchRows * 128;       // 128 channels x 64 fp16 (hi or lo)
    static constexpr int kABufBytes = 2 * kATileBytes;          // hi, then lo
    static constexpr int kXOff = 0;
    static constexpr int kAOff = kSearchXStages * kXStageBytes;
    static constexpr int kBarOff = kAOff + kSearchABufs * kABufBytes;
    static constexpr int kNumBars = 2 * kSearchXStages + 2 * kSearchABufs + 1;
    static constexpr int kRedOff = kBarOff + kNumBars * 8;      // [kSearchProducerWarps] double
    static constexpr int kTmemPtrOff = kRedOff + kSearchProducerWarps * 8;
    static constexpr int kSmemBytes = kTmemPtrOff + 16 + 1024;  // + slack to align the base to 1024
};

// Scratch of one search.  `slots` alpha tables (s as fp32, fl(1/s) 2^e) are held at a
// time: all of them for awq_scale_search, one for the chunked form.
struct SearchWorkspace {
    double* colsum;      // [K]          } zeroed together
    double* wcolsum;     // [K] sum_n |W[n][k]| (duo scaling)
    uint32_t* bound;     // [64] float bits, atomicMax
    uint32_t* wgmax;     // [ng] float bits, atomicMax
    size_t zero_bytes;
    uint16_t* s_all;     // [64][K] fp16
    int32_t* eexp;       // [64]
    double* losses;      // [64]
    float* s32;          // [slots][K]
    float* rse;          // [slots][K]
    double* partial;     // [partial_cap]
    size_t partial_cap;
    size_t bytes;
};

inline size_t search_tiles(int M, int N) {
    return (size_t)ceil_div(N, kSearchRows) * (size_t)ceil_div(M, kSearchTokChunk);
}

inline SearchWorkspace search_layout(void* base, int K, int G, int slots, size_t partial_cap) {
    SearchWorkspace w = {};
    size_t off = 0;
    char* b = static_cast<char*>(base);
    auto take = [&](size_t bytes) {
        char* p = b ? b + off : nullptr;
        off += align256(bytes);
        return p;
    };
    const int ng = K / G;
    w.zero_bytes = (size_t)K * 16 + kSearchMaxGrid * 4 + (size_t)ng * 4;
    w.colsum = reinterpret_cast<double*>(take(w.zero_bytes));
    w.wcolsum = w.colsum + K;
    w.bound = reinterpret_cast<uint32_t*>(w.wcolsum + K);
    w.wgmax = w.bound + kSearchMaxGrid;
    if (!b) w.wcolsum = nullptr, w.bound = w.wgmax = nullptr;
    w.s_all = reinterpret_cast<uint16_t*>(take((size_t)kSearchMaxGrid * K * 2));
    w.eexp = reinterpret_cast<int32_t*>(take(kSearchMaxGrid * 4));
    w.losses = reinterpret_cast<double*>(take(kSearchMaxGrid * 8));
    w.s32 = reinterpret_cast<float*>(take((size_t)slots * K * 4));
    w.rse = reinterpret_cast<float*>(take((size_t)slots * K * 4));
    w.partial_cap = partial_cap;
    w.partial = reinterpret_cast<double*>(take(partial_cap * 8));
    w.bytes = off;
    return w;
}

inline size_t search_workspace_bytes(int M, int N, int K, int G, int /*n_grid*/) {
    if (M <= 0 || N <= 0 || K <= 0 || G <= 0) return 0;
    return search_layout(nullptr, K, G, kSearchMaxGrid, (size_t)kSearchMaxGrid * search_tiles(M, N)).bytes;
}

// ---------------------------------------------------------------------------
// Statistics: max|W| per group over all rows; s per alpha with its group extremes.
// ---------------------------------------------------------------------------

// wgmax[g] = max over every row and the group's channels of |W| (as float bits).  Block:
// 256 threads x 8 channels of a 2048-channel chunk, 64 rows; the G/8 lanes of a group
// reduce by shuffles, one atomic per group and block.
__global__ void __launch_bounds__(256)
group_absmax_kernel(const uint16_t* __restrict__ W, int N, int K, int G, uint32_t* __restrict__ wgmax) {
    const int c0 = blockIdx.x * 2048 + threadIdx.x * 8;
    const int r0 = blockIdx.y * 64;
    const int r1 = min(N, r0 + 64);
    uint32_t m = 0;   // fp16 magnitude bits order like the magnitudes
    if (c0 < K) {
        for (int r = r0; r < r1; ++r) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(W + (size_t)r * K + c0));
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) m = max(m, max(wv[i] & 0x7FFFu, (wv[i] >> 16) & 0x7FFFu));
        }
    }
    for (int off = (G >> 3) >> 1; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (c0 < K && (c0 % G) == 0) atomicMax(wgmax + c0 / G, __float_as_uint(h2f((uint16_t)m)));
}

// For alpha a = a0 + blockIdx.y and group blockIdx.x (blockDim.x = G threads, one channel
// each), with m = colsum / M:
//   plain (wcolsum NULL): s = fp16(max(pow(m, alpha), 2^-14))
//   duo (w = wcolsum / N): s = fp16(min(max(max(pow(m, alpha), 2^-14) /
//                                           max(pow(w, 1 - alpha), 2^-14), 2^-14), 65504))
// all in fp64 with one rounding to fp16, into s_all[a] and (as fp32) into table slot
// blockIdx.y; and the group's term of the bound B into bound[a].
__global__ void search_scales_kernel(const double* __restrict__ colsum, int M, const double* __restrict__ wcolsum,
                                     int N, int K, int n_grid, int a0, const uint32_t* __restrict__ wgmax,
                                     uint16_t* __restrict__ s_all, float* __restrict__ s32,
                                     uint32_t* __restrict__ bound) {
    __shared__ float red[2][8];
    constexpr double kSMin = 6.103515625e-05;   // 2^-14
    const int G = blockDim.x;
    const int g = blockIdx.x, y = blockIdx.y, a = a0 + y;
    const int k = g * G + threadIdx.x;
    const double m = __ddiv_rn(colsum[k], (double)M);
    const double alpha = __ddiv_rn((double)a, (double)n_grid);
    double p = fmax(pow(m, alpha), kSMin);
    if (wcolsum != nullptr) {
        const double w = __ddiv_rn(wcolsum[k], (double)N);
        const double q = fmax(pow(w, __dsub_rn(1.0, alpha)), kSMin);
        p = fmin(fmax(__ddiv_rn(p, q), kSMin), 65504.0);
    }
    const uint16_t h = d2h_rn(p);
    s_all[(size_t)a * K + k] = h;
    const float sf = h2f(h);
    s32[(size_t)y * K + k] = sf;
    float lo = sf, hi = sf;
    for (int off = 16; off > 0; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    const int wid = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[0][wid] = lo, red[1][wid] = hi;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < (G >> 5); ++i) lo = fminf(lo, red[0][i]), hi = fmaxf(hi, red[1][i]);
        const float wm = __uint_as_float(wgmax[g]);
        const float b = __fdiv_ru(__fadd_ru(__fmul_ru(__fmul_ru(3.01f, wm), hi), 1.6e-4f), lo);
        atomicMax(bound + a, __float_as_uint(b));
    }
}

// The exponent of alpha a from its bound (2^e B in [2^14, 2^15)), and the per-channel
// factor rse = fl(1/s) 2^e of table slot blockIdx.y.
__global__ void search_rse_kernel(const float* __restrict__ s32, const uint32_t* __restrict__ bound, int K, int a0,
                                  float* __restrict__ rse, int32_t* __restrict__ eexp) {
    const int y = blockIdx.y, a = a0 + y;
    const float B = __uint_as_float(bound[a]);
    int e = 0;
    if (B > 0.0f && B <= 3.0e38f) {
        int ex;
        frexpf(B, &ex);               // B = f 2^ex, f in [0.5, 1)
        e = min(max(15 - ex, -100), 100);
    }
    const float p2 = __int_as_float((127 + e) << 23);
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x)
        rse[(size_t)y * K + k] = __fmul_rn(__frcp_rn(s32[(size_t)y * K + k]), p2);
    if (blockIdx.x == 0 && threadIdx.x == 0) eexp[a] = e;
}

// ---------------------------------------------------------------------------
// The fused kernel: dW tiles in the producer, E = X dW^T on tcgen05, sum of E^2.
// grid = (row blocks of 128, alphas, token chunks of 512).
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int G>
__global__ void __launch_bounds__(kSearchThreads, 1)
search_fused_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t* __restrict__ W, int M, int N, int K,
                    int zero_point, const uint16_t* __restrict__ s_all, const float* __restrict__ rse,
                    const int32_t* __restrict__ eexp, int a0, double* __restrict__ partial) {
    using C = FusedSearchCfg;
    using namespace sm100;
    constexpr int U = G >= 64 ? G / 64 : 1;      // 64-channel blocks per parameter unit
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* xfull = bars;                               // [kSearchXStages]
    uint64_t* xempty = xfull + kSearchXStages;            // [kSearchXStages]
    uint64_t* afull = xempty + kSearchXStages;            // [kSearchABufs]
    uint64_t* aempty = afull + kSearchABufs;              // [kSearchABufs]
    uint64_t* tfull = aempty + kSearchABufs;
    double* red = reinterpret_cast<double*>(smem + C::kRedOff);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::kTmemPtrOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kSearchRows;
    const int y = blockIdx.y;
    const int m0 = blockIdx.z * kSearchTokChunk;
    const int T = M - m0 > kSearchTokTile ? 2 : 1;        // 256-token accumulators in use
    const uint32_t tcols = T == 2 ? 512u : 256u;
    const int num_kb = ceil_div(K, 64);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSearchXStages; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int b = 0; b < kSearchABufs; ++b) {
            mbar_init(&afull[b], kSearchProducerWarps);
            mbar_init(&aempty[b], 1);
        }
        mbar_init(tfull, 1);
        mbar_fence_init();
        prefetch_tensormap(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA: X tiles [256 tokens x 64 channels], T per stage ----------------
            int issued = 0;
            bool ok = true;
            for (int kb = 0; kb < num_kb && ok; ++kb) {
                const int s = kb % kSearchXStages;
                if (kb >= kSearchXStages) ok = mbar_wait(&xempty[s], ((kb / kSearchXStages) - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&xfull[s], (uint32_t)(T * C::kXTileBytes));
                for (int t = 0; t < T; ++t)
                    tma_load_2d(smem + C::kXOff + s * C::kXStageBytes + t * C::kXTileBytes, &tmap_x, &xfull[s],
                                kb * 64, m0 + t * kSearchTokTile);
                ++issued;
            }
            for (int kb = issued - 1; kb >= 0 && kb >= issued - kSearchXStages; --kb)
                mbar_wait(&xfull[kb % kSearchXStages], (kb / kSearchXStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA: per 16 channels, hi then lo into each accumulator ----------------
            constexpr uint32_t idesc = idesc_f16_f32(kSearchRows, kSearchTokTile);
            bool ok = true;
            for (int kb = 0; kb < num_kb && ok; ++kb) {
                const int s = kb % kSearchXStages, b = kb % kSearchABufs;
                ok = mbar_wait(&xfull[s], (kb / kSearchXStages) & 1) && mbar_wait(&afull[b], (kb / kSearchABufs) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t abase = smem_u32(smem + C::kAOff + b * C::kABufBytes);
                const uint64_t ah = desc_sw128_kmajor(abase), al = desc_sw128_kmajor(abase + C::kATileBytes);
                const uint32_t xbase = smem_u32(smem + C::kXOff + s * C::kXStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    for (int t = 0; t < T; ++t) {
                        const uint64_t bd = desc_sw128_kmajor(xbase + t * C::kXTileBytes);
                        const uint32_t d = tmem + (uint32_t)(t * kSearchTokTile);
                        mma_f16(d, ah + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                        mma_f16(d, al + 2 * kk, bd + 2 * kk, idesc, 1u);
                    }
                }
                mma_commit(&xempty[s]);
                mma_commit(&aempty[b]);
            }
            mma_commit(tfull);   // also on the error path, so that the MMAs drain before TMEM is freed
            if (!ok) mbar_wait(tfull, 0);
        }
    } else {
        // ---------------- producers: dW hi/lo tiles, then the epilogue ----------------
        const int pw = warp - 2;                     // 0..15
        const int d = threadIdx.x - 64;              // 0..511
        const int r = d >> 2;                        // channel row of the tile
        const int qq = d & 3;                        // which 16 channels of a 64-channel block
        const int n = n0 + r;
        const bool row_ok = n < N;
        const bool zp = zero_point != 0;
        const uint16_t* wrow = W + (size_t)(row_ok ? n : 0) * K;
        const uint16_t* sa = s_all + (size_t)(a0 + y) * K;     // s of this alpha, fp16
        const float* ra = rse + (size_t)y * K;
        bool ok = true;
        int produced = 0;
        for (int kb0 = 0; kb0 < num_kb && ok; kb0 += U) {
            // the next unit's lines of W, s and rse into L1 while this unit is computed (its
            // loads would otherwise wait on L2 at the top of every unit)
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int k0n = (kb0 + U + j) * 64 + qq * 16;
                if (k0n < K) {
                    if (row_ok) prefetch_l1(wrow + k0n);
                    prefetch_l1(sa + k0n);
                    prefetch_l1(ra + k0n);
                }
            }
            // pass 1: the unit's weights (kept packed) and the group's extremes of W s
            uint32_t wpk[U][8];
            float mx = -INFINITY, mn = INFINITY;
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int k0 = (kb0 + j) * 64 + qq * 16;
                const bool live = row_ok && k0 < K;
                uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
                if (live) {
                    v0 = __ldg(reinterpret_cast<const uint4*>(wrow + k0));
                    v1 = __ldg(reinterpret_cast<const uint4*>(wrow + k0 + 8));
                }
                wpk[j][0] = v0.x, wpk[j][1] = v0.y, wpk[j][2] = v0.z, wpk[j][3] = v0.w;
                wpk[j][4] = v1.x, wpk[j][5] = v1.y, wpk[j][6] = v1.z, wpk[j][7] = v1.w;
                if (k0 < K) {
                    const uint4 s0 = __ldg(reinterpret_cast<const uint4*>(sa + k0));
                    const uint4 s1 = __ldg(reinterpret_cast<const uint4*>(sa + k0 + 8));
                    const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        float a, b;
                        mul_f16x2_f32(wpk[j][h], sw[h], a, b);                  // W s, exact
                        mx = fmax3(mx, a, b);
                        mn = fmin3(mn, a, b);
                    }
                } else {
                    mx = fmaxf(mx, 0.0f);
                    mn = fminf(mn, 0.0f);
                }
            }
            // a group is 2 lanes (G = 32) or the 4 lanes of the row (G >= 64)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
            if (G >= 64) {
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
            }
            const GroupParams p = group_params(mx, mn, zp);
            const float lo_c = zp ? -p.zero : -8.0f, hi_c = zp ? 15.0f - p.zero : 7.0f;
            const float half_sc = 0.5f * p.sc;
            // pass 2: codes, dW 2^e, the hi/lo split, one 64-channel block at a time
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int kb = kb0 + j;
                if (kb >= num_kb) break;
                const int b = produced % kSearchABufs;
                if (produced >= kSearchABufs) ok = mbar_wait(&aempty[b], ((produced / kSearchABufs) - 1) & 1);
                if (!ok) break;
                const int k0 = kb * 64 + qq * 16;
                uint32_t hw[8], lw[8];
                if (k0 < K) {
                    float ws[16], rr[16];
                    bool good = true;
                    const uint4 s0 = __ldg(reinterpret_cast<const uint4*>(sa + k0));
                    const uint4 s1 = __ldg(reinterpret_cast<const uint4*>(sa + k0 + 8));
                    const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                    for (int h = 0; h < 8; ++h) mul_f16x2_f32(wpk[j][h], sw[h], ws[2 * h], ws[2 * h + 1]);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        // candidate code offset r = rint(ws rc); the residual r sc - ws is exact
                        // while below sc/2, and then rint(fl(ws / sc)) = r is certain
                        rr[i] = rint_magic(__fmul_rn(ws[i], p.rc));
                        const float dd = __fmaf_rn(rr[i], p.sc, -ws[i]);
                        good = good && (__fmaf_rn(fabsf(ws[i]), 0x1p-22f, fabsf(dd)) < half_sc);
                    }
                    if (!good) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) rr[i] = rintf(__fdiv_rn(ws[i], p.sc));
                    }
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const float4 rv = __ldg(reinterpret_cast<const float4*>(ra + k0) + i4);
                        const float r4[4] = {rv.x, rv.y, rv.z, rv.w};
                        float v[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = i4 * 4 + e;
                            const float qz = fminf(fmaxf(rr[i], lo_c), hi_c);        // q - zero
                            const float diff = __fmaf_rn(qz, p.sc, -ws[i]);           // deq - ws
                            v[e] = __fmul_rn(diff, r4[e]);                            // dW 2^e
                        }
#pragma unroll
                        for (int e = 0; e < 4; e += 2) {
                            const uint32_t h2 = pack_f16x2(v[e], v[e + 1]);
                            const float h0 = h2f((uint16_t)(h2 & 0xFFFFu)), h1 = h2f((uint16_t)(h2 >> 16));
                            hw[(i4 * 4 + e) >> 1] = h2;
                            lw[(i4 * 4 + e) >> 1] = pack_f16x2(__fsub_rn(v[e], h0), __fsub_rn(v[e + 1], h1));
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) hw[i] = lw[i] = 0u;
                }
                uint8_t* atile = smem + C::kAOff + b * C::kABufBytes;
                *reinterpret_cast<uint4*>(atile + sw128_offset(r, qq * 2)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(atile + sw128_offset(r, qq * 2 + 1)) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
                *reinterpret_cast<uint4*>(atile + C::kATileBytes + sw128_offset(r, qq * 2)) =
                    make_uint4(lw[0], lw[1], lw[2], lw[3]);
                *reinterpret_cast<uint4*>(atile + C::kATileBytes + sw128_offset(r, qq * 2 + 1)) =
                    make_uint4(lw[4], lw[5], lw[6], lw[7]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&afull[b]);
                ++produced;
            }
        }
        // ---------------- epilogue: sum over this CTA of (E 2^-e)^2 ----------------
        double acc = 0.0;
        if (ok && mbar_wait(tfull, 0)) {
            tc_fence_after();
            const int q4 = warp & 3;                       // TMEM lane quarter of this warp
            const int set = pw >> 2;                       // 0..3: four warps per lane quarter
            const int cols = T * kSearchTokTile / 4;
            const double undo = ldexp(1.0, -eexp[a0 + y]);
            for (int c = set * cols; c < set * cols + cols; c += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)c, v);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const double e = (double)__uint_as_float(v[jj]) * undo;
                    acc = fma(e, e, acc);
                }
            }
        }
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) red[pw] = acc;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int i = 0; i < kSearchProducerWarps; ++i) t += red[i];
        partial[((size_t)y * gridDim.x + blockIdx.x) * gridDim.z + blockIdx.z] = t;
    }
}

// losses[a] = (sum over tiles, fixed order) / (M N)
__global__ void search_loss_kernel(const double* __restrict__ partial, int tiles, double inv_mn,
                                   double* __restrict__ losses) {
    __shared__ double sh[256];
    const int a = blockIdx.x;
    double acc = 0.0;
    for (int i = threadIdx.x; i < tiles; i += 256) acc += partial[(size_t)a * tiles + i];
    sh[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) losses[a] = sh[0] * inv_mn;
}

// losses[0] = (first ? 0 : losses[0]) + sum of the tile partials; * scale when last.
__global__ void search_accum_kernel(const double* __restrict__ partial, int tiles, int first, int last, double scale,
                                    double* __restrict__ loss) {
    __shared__ double sh[256];
    double acc = 0.0;
    for (int i = threadIdx.x; i < tiles; i += 256) acc += partial[i];
    sh[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        double v = (first ? 0.0 : *loss) + sh[0];
        if (last) v *= scale;
        *loss = v;
    }
}

// argmin (ties to the smaller alpha), then s_out = s of the best alpha.
__global__ void search_select_kernel(const double* __restrict__ losses, int n_grid, const uint16_t* __restrict__ s_all,
                                     int K, uint16_t* __restrict__ s_out, int32_t* __restrict__ best_out,
                                     double* __restrict__ losses_out) {
    int best = 0;
    double bl = losses[0];
    for (int i = 1; i < n_grid; ++i)
        if (losses[i] < bl) {
            bl = losses[i];
            best = i;
        }
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k < K) s_out[k] = s_all[(size_t)best * K + k];
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (best_out) *best_out = best;
    }
    if (blockIdx.x == 0 && losses_out && threadIdx.x < n_grid) losses_out[threadIdx.x] = losses[threadIdx.x];
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

inline const void* search_fused_fn(int G) {
    switch (G) {
        case 32: return (const void*)search_fused_kernel<32>;
        case 64: return (const void*)search_fused_kernel<64>;
        case 128: return (const void*)search_fused_kernel<128>;
        default: return (const void*)search_fused_kernel<256>;
    }
}

// Launch of the fused kernel over rows [0, N) of W (already offset by the caller) for
// `count` alphas starting at a0 (their tables in slots 0 .. count-1).
inline awq_status launch_search_fused(const CUtensorMap& tx, const uint16_t* W, int M, int N, int K, int G, int zp,
                                      const SearchWorkspace& w, int a0, int count, cudaStream_t st) {
    const void* fn = search_fused_fn(G);
    if (!prepare_kernel(fn)) return AWQ_ERR_CUDA;
    // carve out no more shared memory than the block needs (196 of 228 KB), so that L1
    // keeps room for the producers' prefetched lines (one unit: up to 33 KB at G = 128)
    if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 86) != cudaSuccess)
        return AWQ_ERR_CUDA;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(ceil_div(N, kSearchRows), count, ceil_div(M, kSearchTokChunk));
    lc.blockDim = dim3(kSearchThreads);
    lc.dynamicSmemBytes = FusedSearchCfg::kSmemBytes;
    lc.stream = st;
    const uint16_t* s_all = w.s_all;
    const float* rse = w.rse;
    const int32_t* eexp = w.eexp;
    double* partial = w.partial;
    void* args[] = {const_cast<CUtensorMap*>(&tx), &W, &M, &N, &K, &zp, &s_all, &rse, &eexp, &a0, &partial};
    return cudaLaunchKernelExC(&lc, fn, args) == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// Statistics shared by both forms: colsum of |X|, max|W| per group (both zeroed first).
inline awq_status search_statistics(const uint16_t* X, int M, const uint16_t* W, int N, int K, int G, bool duo,
                                    const SearchWorkspace& w, cudaStream_t st) {
    if (cudaMemsetAsync(w.colsum, 0, w.zero_bytes, st) != cudaSuccess) return AWQ_ERR_CUDA;
    abs_colsum_kernel<<<dim3(ceil_div(K / 8, 128), (unsigned)min(M, 64)), 128, 0, st>>>(X, M, K, w.colsum);
    if (duo) abs_colsum_kernel<<<dim3(ceil_div(K / 8, 128), (unsigned)min(N, 64)), 128, 0, st>>>(W, N, K, w.wcolsum);
    group_absmax_kernel<<<dim3(ceil_div(K, 2048), ceil_div(N, 64)), 256, 0, st>>>(W, N, K, G, w.wgmax);
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

inline awq_status run_scale_search(const uint16_t* X, int M, const uint16_t* W, int N, int K, int G, int zp,
                                   bool duo, int n_grid, uint16_t* s_out, double* losses_out, int32_t* best_out,
                                   void* ws, cudaStream_t st) {
    const size_t tiles = search_tiles(M, N);
    const SearchWorkspace w = search_layout(ws, K, G, kSearchMaxGrid, (size_t)kSearchMaxGrid * tiles);
    awq_status rc = search_statistics(X, M, W, N, K, G, duo, w, st);
    if (rc != AWQ_OK) return rc;
    search_scales_kernel<<<dim3(K / G, n_grid), G, 0, st>>>(w.colsum, M, duo ? w.wcolsum : nullptr, N, K, n_grid, 0,
                                                            w.wgmax, w.s_all, w.s32, w.bound);
    search_rse_kernel<<<dim3(ceil_div(K, 256), n_grid), 256, 0, st>>>(w.s32, w.bound, K, 0, w.rse, w.eexp);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
    CUtensorMap tx;
    if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)M, (uint64_t)K, kSearchTokTile, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    rc = launch_search_fused(tx, W, M, N, K, G, zp, w, 0, n_grid, st);
    if (rc != AWQ_OK) return rc;
    search_loss_kernel<<<n_grid, 256, 0, st>>>(w.partial, (int)tiles, 1.0 / ((double)M * (double)N), w.losses);
    search_select_kernel<<<ceil_div(K, 256), 256, 0, st>>>(w.losses, n_grid, w.s_all, K, s_out, best_out, losses_out);
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// The same search on scratch of bounded size: one alpha at a time (one table slot), and
// the output channels in chunks whose tile partials fit; each chunk's partials are added
// to the running loss in a fixed order (deterministic).  Used by awq_scale_search_noalloc.
// ---------------------------------------------------------------------------

struct ChunkedSearchLayout {
    SearchWorkspace w;
    int nc;              // output channels per chunk (multiple of kSearchRows); 0 if nothing fits
};

inline ChunkedSearchLayout chunked_search_layout(void* base, size_t bytes, int M, int N, int K, int G) {
    ChunkedSearchLayout L = {};
    const size_t fixed = search_layout(nullptr, K, G, 1, 0).bytes + 256;
    if (fixed >= bytes) return L;
    const size_t cap = (bytes - fixed) / 8;
    const size_t tchunks = (size_t)ceil_div(M, kSearchTokChunk);
    size_t blocks = cap / tchunks;
    const size_t need = (size_t)ceil_div(N, kSearchRows);
    if (blocks > need) blocks = need;
    if (blocks == 0) return L;
    L.w = search_layout(base, K, G, 1, blocks * tchunks);
    if (L.w.bytes > bytes) return L;
    L.nc = (int)(blocks * kSearchRows);
    return L;
}

inline awq_status run_scale_search_chunked(const uint16_t* X, int M, const uint16_t* W, int N, int K, int G, int zp,
                                           int n_grid, uint16_t* s_out, double* losses_out, int32_t* best_out,
                                           const ChunkedSearchLayout& L, cudaStream_t st) {
    if (L.nc <= 0) return AWQ_ERR_UNSUPPORTED;
    const SearchWorkspace& w = L.w;
    awq_status rc = search_statistics(X, M, W, N, K, G, false, w, st);
    if (rc != AWQ_OK) return rc;
    CUtensorMap tx;
    if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)M, (uint64_t)K, kSearchTokTile, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    const double inv_mn = 1.0 / ((double)M * (double)N);
    for (int a = 0; a < n_grid; ++a) {
        search_scales_kernel<<<dim3(K / G, 1), G, 0, st>>>(w.colsum, M, nullptr, N, K, n_grid, a, w.wgmax, w.s_all,
                                                           w.s32, w.bound);
        search_rse_kernel<<<dim3(ceil_div(K, 256), 1), 256, 0, st>>>(w.s32, w.bound, K, a, w.rse, w.eexp);
        if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
        for (int n0 = 0; n0 < N; n0 += L.nc) {
            const int nc = min(L.nc, N - n0);
            rc = launch_search_fused(tx, W + (size_t)n0 * K, M, nc, K, G, zp, w, a, 1, st);
            if (rc != AWQ_OK) return rc;
            const int tiles = (int)search_tiles(M, nc);
            search_accum_kernel<<<1, 256, 0, st>>>(w.partial, tiles, n0 == 0, n0 + nc >= N, inv_mn, w.losses + a);
            if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
        }
    }
    search_select_kernel<<<ceil_div(K, 256), 256, 0, st>>>(w.losses, n_grid, w.s_all, K, s_out, best_out, losses_out);
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
