// apply_clip: per-group weight clipping chosen by the group's output error, on the
// sm_100a tensor cores.
//
// Source: "AI-Research-SKILLs AWQ advanced usage guide" (lshu.cn), section 校准参数全景:
// apply_clip clips the weights to further reduce the effect of outliers on the
// quantisation error.  With the scale s already chosen (ws = W s, exact in fp32), for
// every output channel n, group g and clip ratio r_j = fl32(1 - j / n_grid),
// j = 0 .. n_clip-1:
//   c      = fl32(r_j * max|ws|_group)
//   Q_j    = the group quantiser applied to clamp(ws, -c, c)
//   dW_j   = Q_j / s - W                                      (the unclipped weights)
//   err    = sum_t (sum_{k in g} X[t][k] dW_j[n][k])^2
// and each group keeps the ratio with the smallest error (ties to the smaller j: less
// clipping), then is quantised clipped at it.
//
// One CTA takes 128 output channels, 512 calibration tokens (256 at G = 256) and a run
// of groups.  For a group its producer warps find the group's extremes once; then for
// each ratio they build dW_j 2^e as fp16 hi + lo tiles (the construction of the fused
// scale search; the exponent comes from the same bound), and one tcgen05.mma chain per
// (group, ratio) puts E = X_g dW_j^T in TMEM: with 512 tokens the same dW tile feeds two
// 256-column accumulators (one per 256 tokens), with 256 tokens two tiles alternate
// between them so that one fills while the other drains.  The producers drain a tile
// after building the next: per row the sum over the tokens of E^2 (fp32 over 16 tokens,
// fp64 beyond), the four warps of a row combined in a fixed order.  The errors of the
// CTA's token chunk go to err_part; a second kernel adds the chunks in a fixed order,
// picks the ratio and packs.

#pragma once

#include "common.cuh"
#include "quantize.cuh"
#include "search.cuh"
#include "sm100.cuh"

namespace awq {

constexpr int kClipMaxRatios = 32;
constexpr int kClipRows = 128;
constexpr int kClipABufs = 2;

// Tokens per CTA: 512 up to G = 128, so that each dW tile (group, ratio) feeds two
// 256-column accumulators (half the producer work per multiply-add of 256 tokens); 256 at
// G = 256, whose X for a group (4 blocks) would not fit twice as long.
__host__ __device__ constexpr int clip_tokens(int G) { return G >= 256 ? 256 : 512; }
constexpr int kClipProducerWarps = 16;
constexpr int kClipThreads = 64 + kClipProducerWarps * 32;

template <int G>
struct ClipCfg {
    static constexpr int kTok = clip_tokens(G);
    static constexpr int kHalves = kTok / 256;                      // 256-column accumulators per tile
    static constexpr int kAccSets = kHalves == 1 ? 2 : 1;           // tiles held in TMEM (512 columns)
    static constexpr int kSub = G >= 64 ? G / 64 : 1;              // 64-channel blocks per group
    static constexpr int kXSlots = G >= 128 ? 1 : 2;                // groups of X held
    static constexpr int kXTileBytes = kTok * 128;                  // kTok tokens x 64 channels
    static constexpr int kXSlotBytes = kSub * kXTileBytes;
    static constexpr int kATileBytes = kClipRows * 128;
    static constexpr int kABufBytes = 2 * kATileBytes;              // hi, lo
    static constexpr int kXOff = 0;
    static constexpr int kAOff = kXSlots * kXSlotBytes;
    static constexpr int kBarOff = kAOff + kClipABufs * kABufBytes;
    // xfull, xempty [kXSlots]; afull, aempty [kClipABufs]; accfull, accempty [kAccSets]; done
    static constexpr int kNumBars = 2 * kXSlots + 2 * kClipABufs + 2 * kAccSets + 1;
    static constexpr int kRedOff = kBarOff + kNumBars * 8;          // [2][128][4] double
    static constexpr int kTmemPtrOff = kRedOff + 2 * kClipRows * 4 * 8;
    static constexpr int kSmemBytes = kTmemPtrOff + 16 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory of one CTA exceeds 227 KB");
};

// s as fp32 and the group extremes of s for the exponent bound (one table slot), for a
// given s (NULL: s = 1).  Block: G threads, one group.
__global__ void clip_scale_table_kernel(const uint16_t* __restrict__ s, int K, const uint32_t* __restrict__ wgmax,
                                        float* __restrict__ s32, uint32_t* __restrict__ bound) {
    __shared__ float red[2][8];
    const int G = blockDim.x;
    const int g = blockIdx.x;
    const int k = g * G + threadIdx.x;
    const float sf = s ? h2f(s[k]) : 1.0f;
    s32[k] = sf;
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
        atomicMax(bound, __float_as_uint(b));
    }
}

__device__ __forceinline__ float clip_ratio(int j, int n_grid) {
    return __double2float_rn(__dsub_rn(1.0, __ddiv_rn((double)j, (double)n_grid)));
}

// grid = (CTAs sharing the units, token chunks of clip_tokens(G)).  A unit is (block of
// 128 output channels, group), in the order block-major; CTA c takes the units
// [c U / P, (c + 1) U / P) of the U = ceil(N / 128) ng, so that the CTAs of a wave get
// equal work whatever the block and group counts.  err_part [token chunk][N][ng][n_clip].
template <int G>
__global__ void __launch_bounds__(kClipThreads, 1)
clip_err_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint16_t* __restrict__ W, int M, int N, int K,
                int zero_point, int n_grid, int n_clip, int n_units, const float* __restrict__ s32,
                const float* __restrict__ rse, const int32_t* __restrict__ eexp, double* __restrict__ err_part) {
    using C = ClipCfg<G>;
    using namespace sm100;
    constexpr int U = C::kSub;
    constexpr int kKSteps = G >= 64 ? 4 : 2;       // k16 steps of one 64-channel block used by a group
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* xfull = bars;
    uint64_t* xempty = xfull + C::kXSlots;
    uint64_t* afull = xempty + C::kXSlots;
    uint64_t* aempty = afull + kClipABufs;
    uint64_t* accfull = aempty + kClipABufs;     // [kAccSets]
    uint64_t* accempty = accfull + C::kAccSets;  // [kAccSets]
    uint64_t* done = accempty + C::kAccSets;     // every MMA of the CTA complete
    double* red = reinterpret_cast<double*>(smem + C::kRedOff);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::kTmemPtrOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u_begin = (int)((long long)blockIdx.x * n_units / gridDim.x);
    const int u_end = (int)((long long)(blockIdx.x + 1) * n_units / gridDim.x);
    const int tc = blockIdx.y;
    const int m0 = tc * C::kTok;
    const int ng = K / G;
    const int n_groups = u_end - u_begin;                // units of this CTA
    const int n_tiles = n_groups * n_clip;
    // group and first output channel of the CTA's unit gi
    auto unit_g = [&](int gi) { return (u_begin + gi) % ng; };
    auto unit_n0 = [&](int gi) { return ((u_begin + gi) / ng) * kClipRows; };

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kXSlots; ++i) {
            mbar_init(&xfull[i], 1);
            mbar_init(&xempty[i], 1);
        }
        for (int b = 0; b < kClipABufs; ++b) {
            mbar_init(&afull[b], kClipProducerWarps);
            mbar_init(&aempty[b], 1);
        }
        for (int b = 0; b < C::kAccSets; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], kClipProducerWarps);
        }
        mbar_init(done, 1);
        mbar_fence_init();
        prefetch_tensormap(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA: X of each group (the 64-channel blocks that hold it) ----------------
            int issued = 0;
            bool ok = true;
            for (int gi = 0; gi < n_groups && ok; ++gi) {
                const int slot = gi % C::kXSlots;
                if (gi >= C::kXSlots) ok = mbar_wait(&xempty[slot], ((gi / C::kXSlots) - 1) & 1);
                if (!ok) break;
                const int kbase = (unit_g(gi) * G) & ~63;
                mbar_arrive_expect_tx(&xfull[slot], (uint32_t)(U * C::kXTileBytes));
                for (int u = 0; u < U; ++u)
                    for (int h = 0; h < C::kHalves; ++h)   // boxes of 256 tokens
                        tma_load_2d(smem + C::kXOff + slot * C::kXSlotBytes + u * C::kXTileBytes + h * 256 * 128,
                                    &tmap_x, &xfull[slot], kbase + u * 64, m0 + h * 256);
                ++issued;
            }
            for (int gi = issued - 1; gi >= 0 && gi >= issued - C::kXSlots; --gi)
                mbar_wait(&xfull[gi % C::kXSlots], (gi / C::kXSlots) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA: one accumulator chain per (group, ratio) ----------------
            constexpr uint32_t idesc = idesc_f16_f32(kClipRows, 256);
            bool ok = true;
            int sub = 0;                                   // A sub-tiles consumed
            for (int t = 0; t < n_tiles && ok; ++t) {
                const int gi = t / n_clip, j = t - gi * n_clip;
                const int slot = gi % C::kXSlots;
                const int acc = t % C::kAccSets;
                if (j == 0) ok = mbar_wait(&xfull[slot], (gi / C::kXSlots) & 1);
                if (ok && t >= C::kAccSets) ok = mbar_wait(&accempty[acc], ((t / C::kAccSets) - 1) & 1);
                if (!ok) break;
                const uint32_t d = tmem + (uint32_t)(acc * C::kHalves * 256);
                const int kk0 = G >= 64 ? 0 : ((unit_g(gi) & 1) * 2);        // G = 32: the half of the block
                for (int u = 0; u < U && ok; ++u, ++sub) {
                    const int b = sub % kClipABufs;
                    ok = mbar_wait(&afull[b], (sub / kClipABufs) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t abase = smem_u32(smem + C::kAOff + b * C::kABufBytes);
                    const uint64_t ah = desc_sw128_kmajor(abase), al = desc_sw128_kmajor(abase + C::kATileBytes);
                    const uint32_t xb = smem_u32(smem + C::kXOff + slot * C::kXSlotBytes + u * C::kXTileBytes);
#pragma unroll
                    for (int kq = 0; kq < kKSteps; ++kq) {
                        const int kk = kk0 + kq;
#pragma unroll
                        for (int h = 0; h < C::kHalves; ++h) {   // the same dW feeds every 256 tokens
                            const uint64_t bd = desc_sw128_kmajor(xb + h * 256 * 128);
                            const uint32_t dh = d + (uint32_t)(h * 256);
                            mma_f16(dh, ah + 2 * kk, bd + 2 * kk, idesc, (u | kq) != 0);
                            mma_f16(dh, al + 2 * kk, bd + 2 * kk, idesc, 1u);
                        }
                    }
                    mma_commit(&aempty[b]);
                }
                if (!ok) break;
                mma_commit(&accfull[acc]);
                if (j == n_clip - 1) mma_commit(&xempty[slot]);
            }
            // every MMA issued must complete before TMEM is freed (also after a time-out)
            mma_commit(done);
            mbar_wait(done, 0);
        }
    } else {
        // ---------------- producers: dW_j tiles per (group, ratio); then drain the previous tile ----------------
        const int pw = warp - 2;
        const int dt = threadIdx.x - 64;               // 0..511
        const int r = dt >> 2;                         // channel row of the tile
        const int qq = dt & 3;                         // quarter of the group's channels in a block
        constexpr int CPT = G >= 64 ? 16 : 8;          // channels of a block per thread
        const bool zp = zero_point != 0;
        const double undo = ldexp(1.0, -eexp[0]);
        const int q4 = warp & 3, set = pw >> 2;
        bool ok = true;
        int sub = 0;

        // drain tile t: rows q4*32 + lane, this warp's quarter of the tile's token columns
        auto drain = [&](int t) {
            constexpr int kCols = C::kTok / 4;
            const int acc = t % C::kAccSets;
            double part = 0.0;
            if (ok) ok = mbar_wait(&accfull[acc], (t / C::kAccSets) & 1);
            if (ok) {
                tc_fence_after();
#pragma unroll 2
                for (int c = 0; c < kCols; c += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(acc * C::kHalves * 256 + set * kCols + c),
                              v);
                    tmem_ld_wait();
                    float f = 0.0f;
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const float e = __uint_as_float(v[jj]);
                        f = fmaf(e, e, f);
                    }
                    part += (double)f;
                }
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            double* rb = red + (size_t)(t & 1) * kClipRows * 4;
            rb[(q4 * 32 + lane) * 4 + set] = part;
            // only the four warps of this TMEM lane quarter meet here (named barrier 2 + q4):
            // the row sums need their four parts, and the buffer of tile t is written again
            // at tile t + 2 only by warps that have passed this barrier at tile t + 1
            asm volatile("bar.sync %0, %1;" ::"r"(2 + q4), "n"(4 * 32) : "memory");
            if (set == 0) {
                const int rr = q4 * 32 + lane;
                const int gi = t / n_clip, j = t - gi * n_clip;
                const int nn = unit_n0(gi) + rr;
                const double* q = rb + rr * 4;
                const double sum = ((q[0] + q[1]) + q[2]) + q[3];
                if (nn < N)
                    err_part[(((size_t)tc * N + nn) * ng + unit_g(gi)) * n_clip + j] = sum * undo * undo;
            }
        };

        for (int gi = 0; gi < n_groups; ++gi) {
            const int g = unit_g(gi);
            const int n = unit_n0(gi) + r;                 // this thread's output channel
            const bool row_ok = n < N;
            const uint16_t* wrow = W + (size_t)(row_ok ? n : 0) * K;
            // pass 1: the group's weights (kept packed), ws extremes
            uint32_t wpk[U][CPT / 2];
            float mx = -INFINITY, mn = INFINITY;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k0 = g * G + u * 64 + qq * CPT;
                if (row_ok) {
#pragma unroll
                    for (int h = 0; h < CPT / 8; ++h) {
                        const uint4 v = __ldg(reinterpret_cast<const uint4*>(wrow + k0 + 8 * h));
                        wpk[u][4 * h] = v.x, wpk[u][4 * h + 1] = v.y, wpk[u][4 * h + 2] = v.z, wpk[u][4 * h + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < CPT / 2; ++i) wpk[u][i] = 0u;
                }
#pragma unroll
                for (int i4 = 0; i4 < CPT / 4; ++i4) {
                    const float4 a4 = __ldg(reinterpret_cast<const float4*>(s32 + k0) + i4);
                    const float s4[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = 4 * i4 + e;
                        const uint32_t word = wpk[u][i >> 1];
                        const float ws = __fmul_rn(h2f((uint16_t)((i & 1) ? (word >> 16) : (word & 0xFFFFu))), s4[e]);
                        mx = fmaxf(mx, ws);
                        mn = fminf(mn, ws);
                    }
                }
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
            const float amax = fmaxf(fabsf(mx), fabsf(mn));
            for (int j = 0; j < n_clip; ++j) {      // no early exit: the drains hold a named barrier
                const int t = gi * n_clip + j;
                const float cl = __fmul_rn(clip_ratio(j, n_grid), amax);
                const GroupParams p = group_params(fminf(fmaxf(mx, -cl), cl), fminf(fmaxf(mn, -cl), cl), zp);
                const float lo_c = zp ? -p.zero : -8.0f, hi_c = zp ? 15.0f - p.zero : 7.0f;
                const float half_sc = 0.5f * p.sc;
#pragma unroll
                for (int u = 0; u < U; ++u, ++sub) {
                    const int b = sub % kClipABufs;
                    if (sub >= kClipABufs) ok = ok && mbar_wait(&aempty[b], ((sub / kClipABufs) - 1) & 1);
                    if (!ok) continue;
                    const int k0 = g * G + u * 64 + qq * CPT;
                    uint32_t hw[CPT / 2], lw[CPT / 2];
                    float rr[CPT];
                    bool good = true;
                    // ws = W s is recomputed below (two instructions) rather than held
                    auto wsv = [&](int i, float sc_i) {
                        const uint32_t word = wpk[u][i >> 1];
                        return __fmul_rn(h2f((uint16_t)((i & 1) ? (word >> 16) : (word & 0xFFFFu))), sc_i);
                    };
#pragma unroll
                    for (int i4 = 0; i4 < CPT / 4; ++i4) {
                        const float4 a4 = __ldg(reinterpret_cast<const float4*>(s32 + k0) + i4);
                        const float s4[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 4 * i4 + e;
                            const float wc = fminf(fmaxf(wsv(i, s4[e]), -cl), cl);     // clipped
                            rr[i] = rint_magic(__fmul_rn(wc, p.rc));
                            const float dd = __fmaf_rn(rr[i], p.sc, -wc);
                            good = good && (__fmaf_rn(fabsf(wc), 0x1p-22f, fabsf(dd)) < half_sc);
                        }
                    }
                    if (!good) {
#pragma unroll
                        for (int i = 0; i < CPT; ++i)
                            rr[i] = rintf(__fdiv_rn(fminf(fmaxf(wsv(i, s32[k0 + i]), -cl), cl), p.sc));
                    }
#pragma unroll
                    for (int i4 = 0; i4 < CPT / 4; ++i4) {
                        const float4 a4 = __ldg(reinterpret_cast<const float4*>(s32 + k0) + i4);
                        const float4 b4 = __ldg(reinterpret_cast<const float4*>(rse + k0) + i4);
                        const float s4[4] = {a4.x, a4.y, a4.z, a4.w};
                        const float r4[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                        for (int e = 0; e < 4; e += 2) {
                            const int i = 4 * i4 + e;
                            float v[2];
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const float qz = fminf(fmaxf(rr[i + h], lo_c), hi_c);
                                v[h] = __fmul_rn(__fmaf_rn(qz, p.sc, -wsv(i + h, s4[e + h])), r4[e + h]);   // (deq - ws) 2^e / s
                            }
                            const uint32_t h2 = pack_f16x2(v[0], v[1]);
                            hw[i >> 1] = h2;
                            lw[i >> 1] = pack_f16x2(__fsub_rn(v[0], h2f((uint16_t)(h2 & 0xFFFFu))),
                                                    __fsub_rn(v[1], h2f((uint16_t)(h2 >> 16))));
                        }
                    }
                    uint8_t* atile = smem + C::kAOff + b * C::kABufBytes;
                    // chunk index within the 128-byte row: G >= 64: 2 chunks per thread at 2qq;
                    // G = 32: the group's half of the block, chunk 4 (g & 1) + qq
                    const int ch0 = G >= 64 ? 2 * qq : 4 * (g & 1) + qq;
#pragma unroll
                    for (int h = 0; h < CPT / 8; ++h) {
                        *reinterpret_cast<uint4*>(atile + sw128_offset(r, ch0 + h)) =
                            make_uint4(hw[4 * h], hw[4 * h + 1], hw[4 * h + 2], hw[4 * h + 3]);
                        *reinterpret_cast<uint4*>(atile + C::kATileBytes + sw128_offset(r, ch0 + h)) =
                            make_uint4(lw[4 * h], lw[4 * h + 1], lw[4 * h + 2], lw[4 * h + 3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&afull[b]);
                }
                if (t >= 1) drain(t - 1);
            }
        }
        if (n_tiles >= 1) drain(n_tiles - 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Per (row, group): the errors of the token chunks added in order, the ratio with the
// smallest (ties to the smaller j), then the group quantised clipped at it and packed.
// One block per (4 rows, 2048-channel chunk), as quantize_pack_kernel.
__global__ void __launch_bounds__(kQuantThreads)
clip_pack_kernel(const uint16_t* __restrict__ W, const uint16_t* __restrict__ s, int N, int K, int G, int zero_point,
                 int n_grid, int n_clip, int tchunks, const double* __restrict__ err_part,
                 uint32_t* __restrict__ qweight, uint16_t* __restrict__ scales, uint32_t* __restrict__ qzeros,
                 uint8_t* __restrict__ clip_out, double* __restrict__ err_out) {
    __shared__ uint8_t zbuf[kQuantRows][kQuantChunk / 32];
    const int nchunks = ceil_div(K, kQuantChunk);
    const int row0 = (blockIdx.x / nchunks) * kQuantRows;
    const int chunk = blockIdx.x % nchunks;
    const int k0 = chunk * kQuantChunk + threadIdx.x * 8;
    const bool active = k0 < K;
    const bool zp = zero_point != 0;
    const int ng = K / G;
    float sf[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sf[i] = 1.0f;
    if (s != nullptr && active) {
        const uint4 sv = *reinterpret_cast<const uint4*>(s + k0);
        const uint16_t* sh = reinterpret_cast<const uint16_t*>(&sv);
#pragma unroll
        for (int i = 0; i < 8; ++i) sf[i] = h2f(sh[i]);
    }
    for (int rr = 0; rr < kQuantRows; ++rr) {
        const int row = row0 + rr;
        uint4 wv = make_uint4(0u, 0u, 0u, 0u);
        if (active && row < N) wv = *reinterpret_cast<const uint4*>(W + (size_t)row * K + k0);
        const uint16_t* wh = reinterpret_cast<const uint16_t*>(&wv);
        float ws[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) ws[i] = __fmul_rn(h2f(wh[i]), sf[i]);
        float mx = ws[0], mn = ws[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            mx = fmaxf(mx, ws[i]);
            mn = fminf(mn, ws[i]);
        }
        seg_minmax(mx, mn, G >> 3);
        // the chosen ratio of this group
        int jb = 0;
        if (active && row < N) {
            const int g = k0 / G;
            double best = 0.0;
            const bool writer = err_out != nullptr && (k0 % G) == 0;
            for (int j = 0; j < n_clip; ++j) {
                double e = 0.0;
                for (int c = 0; c < tchunks; ++c) e += err_part[(((size_t)c * N + row) * ng + g) * n_clip + j];
                if (j == 0 || e < best) best = e, jb = j;
                if (writer) err_out[((size_t)row * ng + g) * n_clip + j] = e;
            }
        }
        const float amax = fmaxf(fabsf(mx), fabsf(mn));
        const float cl = __fmul_rn(clip_ratio(jb, n_grid), amax);
        const GroupParams p = group_params(fminf(fmaxf(mx, -cl), cl), fminf(fmaxf(mn, -cl), cl), zp);
        if (active && row < N) {
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) word |= quant_code(fminf(fmaxf(ws[i], -cl), cl), p, zp) << code_shift(i);
            qweight[(size_t)row * (K >> 3) + (k0 >> 3)] = word;
            if ((k0 % G) == 0) {
                const int g = k0 / G;
                scales[(size_t)row * ng + g] = p.sc16;
                zbuf[rr][(threadIdx.x * 8) / G] = (uint8_t)p.zero;
                if (clip_out) clip_out[(size_t)row * ng + g] = (uint8_t)jb;
            }
        }
    }
    if (!zp) return;
    __syncthreads();
    const int groups_here = kQuantChunk / G;
    const int g_base = chunk * groups_here;
    const int words = groups_here / 8;
    for (int t = threadIdx.x; t < kQuantRows * words; t += kQuantThreads) {
        const int rr = t / words, zw = t - rr * words;
        const int row = row0 + rr;
        if (row < N && g_base + zw * 8 < ng) {
            uint32_t word = 0;
            for (int i = 0; i < 8; ++i) {
                const int g = g_base + zw * 8 + i;
                if (g < ng) word |= (uint32_t)zbuf[rr][zw * 8 + i] << (4 * i);
            }
            qzeros[(size_t)row * ceil_div(ng, 8) + (g_base >> 3) + zw] = word;
        }
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct ClipWorkspace {
    uint32_t* bound;     // [1]     } zeroed together
    uint32_t* wgmax;     // [ng]    }
    size_t zero_bytes;
    float* s32;          // [K]
    float* rse;          // [K]
    int32_t* eexp;       // [1]
    double* err;         // [tchunks][N][ng][n_clip]
    size_t bytes;
};

inline ClipWorkspace clip_layout(void* base, int M, int N, int K, int G, int n_clip) {
    ClipWorkspace w = {};
    size_t off = 0;
    char* b = static_cast<char*>(base);
    auto take = [&](size_t bytes) {
        char* p = b ? b + off : nullptr;
        off += align256(bytes);
        return p;
    };
    const int ng = K / G;
    w.zero_bytes = 4 + (size_t)ng * 4;
    w.bound = reinterpret_cast<uint32_t*>(take(w.zero_bytes));
    w.wgmax = b ? w.bound + 1 : nullptr;
    w.s32 = reinterpret_cast<float*>(take((size_t)K * 4));
    w.rse = reinterpret_cast<float*>(take((size_t)K * 4));
    w.eexp = reinterpret_cast<int32_t*>(take(4));
    w.err = reinterpret_cast<double*>(take((size_t)ceil_div(M, clip_tokens(G)) * N * ng * n_clip * 8));
    w.bytes = off;
    return w;
}

inline size_t clip_workspace_bytes(int M, int N, int K, int G, int n_clip) {
    if (M <= 0 || N <= 0 || K <= 0 || G <= 0 || n_clip <= 0) return 0;
    return clip_layout(nullptr, M, N, K, G, n_clip).bytes;
}

inline const void* clip_err_fn(int G) {
    switch (G) {
        case 32: return (const void*)clip_err_kernel<32>;
        case 64: return (const void*)clip_err_kernel<64>;
        case 128: return (const void*)clip_err_kernel<128>;
        default: return (const void*)clip_err_kernel<256>;
    }
}

inline size_t clip_smem_bytes(int G) {
    switch (G) {
        case 32: return ClipCfg<32>::kSmemBytes;
        case 64: return ClipCfg<64>::kSmemBytes;
        case 128: return ClipCfg<128>::kSmemBytes;
        default: return ClipCfg<256>::kSmemBytes;
    }
}

inline awq_status run_apply_clip(const uint16_t* X, int M, const uint16_t* W, const uint16_t* s, int N, int K, int G,
                                 int zp, int n_grid, int n_clip, uint32_t* qweight, uint16_t* scales,
                                 uint32_t* qzeros, uint8_t* clip_out, double* err_out, void* ws, cudaStream_t st,
                                 int sms) {
    const ClipWorkspace w = clip_layout(ws, M, N, K, G, n_clip);
    const int ng = K / G;
    if (cudaMemsetAsync(w.bound, 0, w.zero_bytes, st) != cudaSuccess) return AWQ_ERR_CUDA;
    group_absmax_kernel<<<dim3(ceil_div(K, 2048), ceil_div(N, 64)), 256, 0, st>>>(W, N, K, G, w.wgmax);
    clip_scale_table_kernel<<<ng, G, 0, st>>>(s, K, w.wgmax, w.s32, w.bound);
    search_rse_kernel<<<dim3(ceil_div(K, 256), 1), 256, 0, st>>>(w.s32, w.bound, K, 0, w.rse, w.eexp);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
    CUtensorMap tx;
    if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)M, (uint64_t)K, 256, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    const void* fn = clip_err_fn(G);
    if (!prepare_kernel(fn)) return AWQ_ERR_CUDA;
    // the (128-channel block, group) units shared evenly by one wave of CTAs (or all units
    // when there are fewer)
    const int rb = ceil_div(N, kClipRows), tcs = ceil_div(M, clip_tokens(G));
    const int n_units = rb * ng;
    const int ctas = max(1, min(n_units, max(1, sms / tcs)));
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(ctas, tcs);
    lc.blockDim = dim3(kClipThreads);
    lc.dynamicSmemBytes = clip_smem_bytes(G);
    lc.stream = st;
    const float* s32 = w.s32;
    const float* rse = w.rse;
    const int32_t* eexp = w.eexp;
    double* err = w.err;
    int units_arg = n_units;
    void* args[] = {&tx, &W, &M, &N, &K, &zp, &n_grid, &n_clip, &units_arg, &s32, &rse, &eexp, &err};
    if (cudaLaunchKernelExC(&lc, fn, args) != cudaSuccess) return AWQ_ERR_CUDA;
    const long long blocks = (long long)ceil_div(N, kQuantRows) * ceil_div(K, kQuantChunk);
    clip_pack_kernel<<<(unsigned)blocks, kQuantThreads, 0, st>>>(W, s, N, K, G, zp, n_grid, n_clip, tcs, w.err,
                                                                qweight, scales, zp ? qzeros : nullptr, clip_out,
                                                                err_out);
    stream_order_kernel<<<1, 32, 0, st>>>();
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
