// Fused dequantising W4A16 GEMM on the sm_100a tensor cores (tcgen05 + TMA + TMEM).
//
// Source: "Optimization Awq" (skillsdirectory.com), kernel backends: GEMM is the
// default for batch sizes > 1 (batched decode and prefill); "AI-Research-SKILLs AWQ
// advanced usage guide" (lshu.cn), WQLinear kernels.  Result as the header defines:
// Y[m][n] = sum_k X[m][k] * (q[n][k] - z[n][g]) * scale16[n][g], fp32 accumulation.
//
// Formulation.  The kernel computes Y^T tile by tile: D[n][m] = sum_k Wdeq[n][k] X[m][k]
// with the dequantised weight tile as the MMA's A operand (M_mma = 128 output
// channels) and the activations as B (N_mma = BN tokens, 16..256).  Each weight tile
// is dequantised once per CTA and reused for BN tokens, so the dequant work per
// multiply-add is 1/BN, and small token counts use a narrow MMA instead of padding.
//
// Warp roles (608 threads):
//   warp 0      TMA producer of X: tile [BN x 64] fp16 (128B swizzle) per 64-channel k-block,
//               into a ring whose slots the MMAs free.
//   warp 1      allocates TMEM; one lane issues 4 tcgen05.mma (K = 16 each) per k-block.
//   warp 2      TMA producer of the packed weights: tile [128 rows x 32 words] = 4 k-blocks per
//               stage (a whole 128-byte line per row; with one 32-byte row per k-block the
//               copies landed at about 4 B/cycle per SM), 128B-swizzled, into a ring of its
//               own whose slots the dequantisers free as soon as they have read the words,
//               so that refilling it never waits for the MMAs.
//   warps 3..18 dequantise: thread (row, quarter) turns 16 codes per k-block into fp16
//               (q - z) * scale16 with mask/magic-number arithmetic, a batch of k-blocks per
//               iteration, and writes them in the 128B-swizzled K-major layout the MMA
//               reads; afterwards they are the epilogue, reading the fp32 accumulator from
//               TMEM and storing fp16 Y (or fp32 partial sums of a K split).
// Every wait is bounded (2 s): on time-out the kernel raises the device error word,
// drains what it issued, frees TMEM and returns.
#pragma once

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace awq {

constexpr int kDequantWarps = 16;
constexpr int kGemmThreads = 96 + kDequantWarps * 32;   // X TMA, MMA, W TMA, dequant/epilogue warps
constexpr int kGemmTileN = 128;      // output channels per CTA (MMA M)
constexpr int kGemmKB = 64;          // input channels per k-block
constexpr int kDequantThreads = kDequantWarps * 32;   // 4 threads per row, 16 codes each

// Byte offset `a` inside a packed-weight stage whose rows are 32 * WKB bytes, as TMA lays it
// out with the 32 * WKB-byte swizzle (none for one k-block): the 16-byte unit index is
// XOR-ed with the 128-byte line index, modulo the swizzle span.  The stage starts on a
// 1024-byte boundary.
template <int WKB>
__device__ __forceinline__ uint32_t wstage_swizzle(uint32_t a) {
    if constexpr (WKB == 1) return a;
    else return a ^ (((a >> 7) & (uint32_t)(2 * WKB - 1)) << 4);
}

template <int BN>
struct GemmCfg {
    static constexpr int kXStages = BN >= 256 ? 4 : (BN >= 64 ? 6 : 8);
    // packed weights: kWKB k-blocks per stage (rows of one 128-byte line)
    static constexpr int kWKB = 4;
    static constexpr int kWStages = BN >= 256 ? 2 : (BN >= 64 ? 3 : 4);
    static constexpr int kABufs = BN >= 256 ? 3 : (BN >= 128 ? 4 : 8);
    // k-blocks a dequantising thread converts per iteration (one fence and one wait per
    // barrier round trip for all of them); half the A buffers, so that the MMA consumes
    // one batch while the next is written
    static constexpr int kBatch = BN >= 256 ? 1 : kABufs / 2;
    static constexpr int kXBytes = BN * 128;                 // X tile: BN rows x 128 B
    static constexpr int kWBytes = kGemmTileN * 32 * kWKB;   // packed stage: 128 rows x 128 B
    static constexpr int kABytes = kGemmTileN * 128;         // dequantised tile
    static constexpr int kXOff = 0;
    static constexpr int kAOff = kXOff + kXStages * kXBytes;  // both multiples of 1024
    static constexpr int kWOff = kAOff + kABufs * kABytes;
    static constexpr int kBarOff = kWOff + kWStages * kWBytes;
    static constexpr int kNumBars = 2 * kXStages + 2 * kWStages + 2 * kABufs + 1;
    static constexpr int kTmemPtrOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kTmemPtrOff + 16 + 1024;   // + slack to align the base to 1024
    static constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
    static_assert(kSmemBytes <= 232448, "shared memory of one CTA exceeds 227 KB");
    static_assert(kXStages >= kBatch && kABufs >= 2 * kBatch || kBatch == 1, "ring depths");
    static_assert(kWKB % kBatch == 0, "a batch of k-blocks lies in one packed-weight stage");
    static_assert(kWKB == 4 && kWOff % 1024 == 0, "128-byte swizzled packed stages on 1024-byte boundaries");
};

// (q - z) * s for the 8 codes of one word, returned as 4 fp16 pairs in k order.  The
// codes k, k+1 of a word sit at the same nibble of its two 16-bit halves, so each mask
// below leaves one adjacent pair, already in order.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t zmagic, uint32_t zneg16, uint32_t s2) {
    const uint32_t kMagic = 0x64006400u;     // fp16 1024 in both halves
    const uint32_t kSixteenth = 0x2C002C00u; // fp16 1/16 in both halves
    uint32_t a = (w & 0x000F000Fu) | kMagic;            // 1024 + q0, 1024 + q1
    uint32_t b = (w & 0x00F000F0u) | kMagic;            // 1024 + 16 q2, 1024 + 16 q3
    const uint32_t w8 = w >> 8;
    uint32_t c = (w8 & 0x000F000Fu) | kMagic;           // q4, q5
    uint32_t d = (w8 & 0x00F000F0u) | kMagic;           // 16 q6, 16 q7
    asm("sub.rn.f16x2 %0, %0, %4;\n\t"                  // q - z (exact)
        "fma.rn.f16x2 %1, %1, %5, %6;\n\t"              // (1024 + 16q)/16 - (64 + z) = q - z (exact)
        "sub.rn.f16x2 %2, %2, %4;\n\t"
        "fma.rn.f16x2 %3, %3, %5, %6;\n\t"
        "mul.rn.f16x2 %0, %0, %7;\n\t"                  // * scale16 (one rounding)
        "mul.rn.f16x2 %1, %1, %7;\n\t"
        "mul.rn.f16x2 %2, %2, %7;\n\t"
        "mul.rn.f16x2 %3, %3, %7;"
        : "+r"(a), "+r"(b), "+r"(c), "+r"(d)
        : "r"(zmagic), "r"(kSixteenth), "r"(zneg16), "r"(s2));
    return make_uint4(a, b, c, d);   // (k0, k1) (k2, k3) (k4, k5) (k6, k7)
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_q,
                  const uint16_t* __restrict__ scales, const uint32_t* __restrict__ qzeros, int M, int N, int K,
                  int G, int zero_point, uint16_t* __restrict__ Y, int kb_per, float* __restrict__ part) {
    using C = GemmCfg<BN>;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* xfull = bars;                         // [kXStages] X landed
    uint64_t* xempty = xfull + C::kXStages;         // [kXStages] MMA done with the X slot
    uint64_t* wfull = xempty + C::kXStages;         // [kWStages] packed tile landed
    uint64_t* wempty = wfull + C::kWStages;         // [kWStages] dequantisers have read it
    uint64_t* afull = wempty + C::kWStages;         // [kABufs]   dequantised tile written
    uint64_t* aempty = afull + C::kABufs;           // [kABufs]   MMA done with the dequantised tile
    uint64_t* tfull = aempty + C::kABufs;           // accumulator complete
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::kTmemPtrOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * BN;
    const int n0 = blockIdx.y * kGemmTileN;
    // split K: this CTA takes k-blocks [kb0, kb0 + num_kb); with part != NULL it writes
    // fp32 partial sums to part[blockIdx.z][M][N] instead of Y
    const int kb0 = blockIdx.z * kb_per;
    const int num_kb = max(0, min(kb_per, ceil_div(K, kGemmKB) - kb0));

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kXStages; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int s = 0; s < C::kWStages; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], kDequantWarps);
        }
        for (int a = 0; a < C::kABufs; ++a) {
            mbar_init(&afull[a], kDequantWarps);
            mbar_init(&aempty[a], 1);
        }
        mbar_init(tfull, 1);
        mbar_fence_init();
        prefetch_tensormap(&tmap_x);
        prefetch_tensormap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0 || warp == 2) {
        if (lane == 0) {
            // ---------------- TMA: X ring (warp 0) or packed-weight ring (warp 2) ----------------
            const bool xs = warp == 0;
            const int S = xs ? C::kXStages : C::kWStages;
            const int n_st = xs ? num_kb : ceil_div(num_kb, C::kWKB);   // one or kWKB k-blocks a stage
            uint64_t* full = xs ? xfull : wfull;
            uint64_t* empty = xs ? xempty : wempty;
            const uint32_t bytes = xs ? C::kXBytes : C::kWBytes;
            uint8_t* base = smem + (xs ? C::kXOff : C::kWOff);
            int issued = 0;
            bool ok = true;
            for (int j = 0; j < n_st && ok; ++j) {
                const int s = j % S;
                if (j >= S) ok = mbar_wait(&empty[s], ((j / S) - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[s], bytes);
                if (xs)
                    tma_load_2d(base + s * bytes, &tmap_x, &full[s], (kb0 + j) * kGemmKB, m0);
                else
                    tma_load_2d(base + s * bytes, &tmap_q, &full[s], (kb0 + j * C::kWKB) * (kGemmKB / 8), n0);
                ++issued;
            }
            // Drain: every issued copy must land before the CTA may exit.
            for (int j = issued - 1; j >= 0 && j >= issued - S; --j) mbar_wait(&full[j % S], (j / S) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t idesc = idesc_f16_f32(kGemmTileN, BN);
            bool ok = true;
            for (int kb = 0; kb < num_kb && ok; ++kb) {
                const int s = kb % C::kXStages;
                const int a = kb % C::kABufs;
                ok = mbar_wait(&xfull[s], (kb / C::kXStages) & 1) && mbar_wait(&afull[a], (kb / C::kABufs) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint64_t adesc = desc_sw128_kmajor(smem_u32(smem + C::kAOff + a * C::kABytes));
                const uint64_t bdesc = desc_sw128_kmajor(smem_u32(smem + C::kXOff + s * C::kXBytes));
#pragma unroll
                for (int kk = 0; kk < kGemmKB / 16; ++kk)
                    mma_f16(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
                mma_commit(&xempty[s]);
                mma_commit(&aempty[a]);
            }
            mma_commit(tfull);   // also on the error path, so that the MMAs drain before TMEM is freed
            if (!ok) mbar_wait(tfull, 0);
        }
    } else {
        // ---------------- dequantise, then epilogue ----------------
        const int d = threadIdx.x - 96;           // 0..511
        const int row = d & (kGemmTileN - 1);
        const int kq = d >> 7;                    // which 16 channels of the k-block
        const int n = n0 + row;
        const int ng = K / G;
        const int nzw = ceil_div(ng, 8);
        const bool zp = zero_point != 0;
        const bool row_ok = n < N;
        const int lg = 31 - __clz(G);             // G is a power of two
        const uint16_t* srow = scales + (size_t)(row_ok ? n : 0) * ng;
        const uint32_t* zrow = qzeros + (size_t)(row_ok ? n : 0) * nzw;
        // scale and zero word of the thread's next group, fetched a group ahead (raw; using
        // a loaded value stalls on its load)
        const int g_first = (kb0 * kGemmKB + kq * 16) >> lg;
        uint32_t sc_next = row_ok ? __ldg(srow + g_first) : 0u;
        uint32_t zw_next = (row_ok && zp) ? __ldg(zrow + (g_first >> 3)) : 0u;
        int g_cur = -1;
        uint32_t s2 = 0, zmagic = 0x64006400u, zneg16 = 0;
        bool ok = true;
        constexpr int D = C::kBatch;
        for (int kb = 0; kb < num_kb && ok; kb += D) {
            // the batch's A buffers free and its packed tiles landed
            uint2 packed[D];
#pragma unroll
            for (int i = 0; i < D; ++i) {
                const int kbi = kb + i;
                packed[i] = make_uint2(0u, 0u);
                if (kbi < num_kb) {
                    if (kbi >= C::kABufs) ok = ok && mbar_wait(&aempty[kbi % C::kABufs], ((kbi / C::kABufs) - 1) & 1);
                    const int j = kbi / C::kWKB, sb = kbi % C::kWKB;   // stage, k-block inside it
                    if (i == 0) ok = ok && mbar_wait(&wfull[j % C::kWStages], (j / C::kWStages) & 1);
                    if (ok)
                        packed[i] = *reinterpret_cast<const uint2*>(
                            smem + C::kWOff + (j % C::kWStages) * C::kWBytes +
                            wstage_swizzle<C::kWKB>(row * (32 * C::kWKB) + sb * 32 + kq * 8));
                }
            }
            if (!ok) break;
#pragma unroll
            for (int i = 0; i < D; ++i) {
                const int kbi = kb + i;
                if (kbi >= num_kb) break;
                const int k = (kb0 + kbi) * kGemmKB + kq * 16;
                const bool live = row_ok && k < K;
                const int g_here = k >> lg;
                if (live && g_here != g_cur) {   // sc_next / zw_next hold this group's parameters
                    g_cur = g_here;
                    const uint32_t sc = sc_next;
                    const uint32_t z = zp ? ((zw_next >> (4 * (g_cur & 7))) & 15u) : 8u;
                    s2 = sc | (sc << 16);
                    const uint32_t zm = 0x6400u | z;                               // 1024 + z
                    zmagic = zm | (zm << 16);
                    const uint32_t zn = 0xD000u | (z << 4) | 0x0400u;              // fp16 -(64 + z): 2^6 * (1 + z/64)
                    zneg16 = zn | (zn << 16);
                    // the fp16 product (q - z) * scale16 is finite for every code of the group
                    // iff max|q - z| * scale16 < 65520 (exact in fp32); otherwise flag it
                    const float qz_max = zp ? fmaxf((float)z, 15.0f - (float)z) : 8.0f;
                    if (!(h2f((uint16_t)sc) * qz_max < 65520.0f) && !isnan(h2f((uint16_t)sc))) raise_error(kErrRange);
                    // the next group this thread reaches (G / 64 k-blocks on, at least one): its
                    // parameters are fetched now, a whole group ahead of their use
                    const int gn = g_cur + (lg >= 6 ? 1 : (kGemmKB >> lg));
                    if ((gn << lg) < K) {
                        sc_next = __ldg(srow + gn);
                        if (zp) zw_next = __ldg(zrow + (gn >> 3));
                    }
                }
                uint8_t* atile = smem + C::kAOff + (kbi % C::kABufs) * C::kABytes;
                const uint4 v0 = live ? dequant_word(packed[i].x, zmagic, zneg16, s2) : make_uint4(0, 0, 0, 0);
                const uint4 v1 = live ? dequant_word(packed[i].y, zmagic, zneg16, s2) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(atile + sw128_offset(row, kq * 2)) = v0;
                *reinterpret_cast<uint4*>(atile + sw128_offset(row, kq * 2 + 1)) = v1;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {   // the packed words have been used: a finished stage goes back to the producer
#pragma unroll
                for (int i = 0; i < D; ++i) {
                    const int kbi = kb + i;
                    if (kbi < num_kb) {
                        if (kbi % C::kWKB == C::kWKB - 1 || kbi == num_kb - 1)
                            mbar_arrive(&wempty[(kbi / C::kWKB) % C::kWStages]);
                        mbar_arrive(&afull[kbi % C::kABufs]);
                    }
                }
            }
        }
        if (ok && mbar_wait(tfull, 0)) {
            tc_fence_after();
            const int q = warp & 3;                        // TMEM lane quarter this warp may access
            const int set = (warp - 3) >> 2;               // 0..3: four warps per lane quarter
            const int cols = BN >= 64 ? BN / 4 : 16;
            const int c_begin = set * cols;
            if (c_begin < BN) {
                const int nn = n0 + q * 32 + lane;
                for (int c = c_begin; c < c_begin + cols; c += 16) {
                    uint32_t r[16];
                    tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, r);
                    tmem_ld_wait();
                    if (nn < N) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int m = m0 + c + j;
                            if (m < M) {
                                if (part)
                                    part[((size_t)blockIdx.z * M + m) * N + nn] = __uint_as_float(r[j]);
                                else
                                    Y[(size_t)m * N + nn] = f2h_rn(__uint_as_float(r[j]));
                            }
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Wide form for prefill (M > 128): 256 output channels x 256 tokens per CTA, two
// dequantised 128-channel A tiles per 64-channel k-block, two 256-column TMEM
// accumulators.  Every X tile then feeds twice the MMA work of the 128-channel form, and
// the packed weights have a ring of their own, freed by the dequantisers, so that the X
// ring (freed by the MMAs) is the only round trip on the MMA's critical path.
//   warp 0     TMA: X tiles [256 tokens x 64] into the X ring
//   warp 1     TMEM allocation; one lane issues 8 tcgen05.mma per k-block
//   warp 2     TMA: packed tiles [256 rows x 8 kWKB words] (kWKB k-blocks) into the W ring
//   warps 3-18 dequantise (thread = row, 32 codes), then the epilogue
// ---------------------------------------------------------------------------
constexpr int kWideRows = 256;
constexpr int kWideBN = 256;
constexpr int kWideThreads = 96 + kDequantWarps * 32;

struct GemmWideCfg {
    // packed weights: kWKB k-blocks per stage, rows of 32 kWKB bytes (swizzled to match)
    static constexpr int kWKB = 1;
    static constexpr int kXStages = kWKB >= 4 ? 3 : 4;
    static constexpr int kWStages = kWKB >= 2 ? 2 : 4;
    static constexpr int kABufs = 2;
    static constexpr int kXBytes = kWideBN * 128;              // 256 tokens x 64 fp16
    static constexpr int kWBytes = kWideRows * 32 * kWKB;      // 256 rows x 8 kWKB words
    static constexpr int kATileBytes = kGemmTileN * 128;       // one 128-channel tile
    static constexpr int kABytes = 2 * kATileBytes;
    static constexpr int kXOff = 0;
    static constexpr int kAOff = kXOff + kXStages * kXBytes;
    static constexpr int kWOff = kAOff + kABufs * kABytes;
    static constexpr int kBarOff = kWOff + kWStages * kWBytes;
    static constexpr int kNumBars = 2 * kXStages + 2 * kWStages + 2 * kABufs + 1;
    static constexpr int kTmemPtrOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kTmemPtrOff + 16 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory of one CTA exceeds 227 KB");
    static_assert((kWKB == 1 || kWKB == 2 || kWKB == 4) && kWOff % 1024 == 0, "swizzled packed stages");
};

__global__ void __launch_bounds__(kWideThreads, 1)
gemm_w4a16_wide_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_q,
                       const uint16_t* __restrict__ scales, const uint32_t* __restrict__ qzeros, int M, int N, int K,
                       int G, int zero_point, uint16_t* __restrict__ Y) {
    using C = GemmWideCfg;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* xfull = bars;                         // [kXStages] X landed
    uint64_t* xempty = xfull + C::kXStages;         // [kXStages] MMA done with the X slot
    uint64_t* wfull = xempty + C::kXStages;         // [kWStages] packed tile landed
    uint64_t* wempty = wfull + C::kWStages;         // [kWStages] dequantisers done with it
    uint64_t* afull = wempty + C::kWStages;         // [kABufs]  dequantised tiles written
    uint64_t* aempty = afull + C::kABufs;           // [kABufs]  MMA done with them
    uint64_t* tfull = aempty + C::kABufs;           // accumulators complete
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::kTmemPtrOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kWideBN;
    const int n0 = blockIdx.y * kWideRows;
    const int num_kb = ceil_div(K, kGemmKB);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kXStages; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int s = 0; s < C::kWStages; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], kDequantWarps);
        }
        for (int a = 0; a < C::kABufs; ++a) {
            mbar_init(&afull[a], kDequantWarps);
            mbar_init(&aempty[a], 1);
        }
        mbar_init(tfull, 1);
        mbar_fence_init();
        prefetch_tensormap(&tmap_x);
        prefetch_tensormap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0 || warp == 2) {
        if (lane == 0) {
            // ---------------- TMA: X ring (warp 0) or packed-weight ring (warp 2) ----------------
            const bool xs = warp == 0;
            const int S = xs ? C::kXStages : C::kWStages;
            const int n_st = xs ? num_kb : ceil_div(num_kb, C::kWKB);   // one or kWKB k-blocks a stage
            uint64_t* full = xs ? xfull : wfull;
            uint64_t* empty = xs ? xempty : wempty;
            const uint32_t bytes = xs ? C::kXBytes : C::kWBytes;
            uint8_t* base = smem + (xs ? C::kXOff : C::kWOff);
            int issued = 0;
            bool ok = true;
            for (int j = 0; j < n_st && ok; ++j) {
                const int s = j % S;
                if (j >= S) ok = mbar_wait(&empty[s], ((j / S) - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[s], bytes);
                if (xs)
                    tma_load_2d(base + s * bytes, &tmap_x, &full[s], j * kGemmKB, m0);
                else
                    tma_load_2d(base + s * bytes, &tmap_q, &full[s], j * C::kWKB * (kGemmKB / 8), n0);
                ++issued;
            }
            for (int j = issued - 1; j >= 0 && j >= issued - S; --j) mbar_wait(&full[j % S], (j / S) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t idesc = idesc_f16_f32(kGemmTileN, kWideBN);
            bool ok = true;
            for (int kb = 0; kb < num_kb && ok; ++kb) {
                const int s = kb % C::kXStages;
                const int a = kb % C::kABufs;
                ok = mbar_wait(&xfull[s], (kb / C::kXStages) & 1) && mbar_wait(&afull[a], (kb / C::kABufs) & 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t abase = smem_u32(smem + C::kAOff + a * C::kABytes);
                const uint64_t a0 = desc_sw128_kmajor(abase), a1 = desc_sw128_kmajor(abase + C::kATileBytes);
                const uint64_t bdesc = desc_sw128_kmajor(smem_u32(smem + C::kXOff + s * C::kXBytes));
#pragma unroll
                for (int kk = 0; kk < kGemmKB / 16; ++kk) {
                    mma_f16(tmem, a0 + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
                    mma_f16(tmem + kWideBN, a1 + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
                }
                mma_commit(&xempty[s]);
                mma_commit(&aempty[a]);
            }
            mma_commit(tfull);   // also on the error path, so that the MMAs drain before TMEM is freed
            if (!ok) mbar_wait(tfull, 0);
        }
    } else {
        // ---------------- dequantise (thread = channel row, 32 codes), then epilogue ----------------
        const int d = threadIdx.x - 96;           // 0..511
        const int row = d & (kWideRows - 1);      // 0..255
        const int kh = d >> 8;                    // which 32 channels of the k-block
        const int rt = row >> 7, r = row & 127;
        const int n = n0 + row;
        const int ng = K / G;
        const int nzw = ceil_div(ng, 8);
        const bool zp = zero_point != 0;
        const bool row_ok = n < N;
        const int lg = 31 - __clz(G);             // G is a power of two
        const uint16_t* srow = scales + (size_t)(row_ok ? n : 0) * ng;
        const uint32_t* zrow = qzeros + (size_t)(row_ok ? n : 0) * nzw;
        const int g_first = (kh * 32) >> lg;
        uint32_t sc_next = row_ok ? __ldg(srow + g_first) : 0u;
        uint32_t zw_next = (row_ok && zp) ? __ldg(zrow + (g_first >> 3)) : 0u;
        int g_cur = -1;
        uint32_t s2 = 0, zmagic = 0x64006400u, zneg16 = 0;
        bool ok = true;
        for (int kb = 0; kb < num_kb && ok; ++kb) {
            const int j = kb / C::kWKB, sb = kb % C::kWKB;   // packed-weight stage, k-block inside it
            const int s = j % C::kWStages;
            const int a = kb % C::kABufs;
            const int k = kb * kGemmKB + kh * 32;
            const bool live = row_ok && k < K;
            const int g_here = k >> lg;
            if (live && g_here != g_cur) {   // sc_next / zw_next hold this group's parameters
                g_cur = g_here;
                const uint32_t sc = sc_next;
                const uint32_t z = zp ? ((zw_next >> (4 * (g_cur & 7))) & 15u) : 8u;
                s2 = sc | (sc << 16);
                const uint32_t zm = 0x6400u | z;
                zmagic = zm | (zm << 16);
                const uint32_t zn = 0xD000u | (z << 4) | 0x0400u;
                zneg16 = zn | (zn << 16);
                const float qz_max = zp ? fmaxf((float)z, 15.0f - (float)z) : 8.0f;
                if (!(h2f((uint16_t)sc) * qz_max < 65520.0f) && !isnan(h2f((uint16_t)sc))) raise_error(kErrRange);
                // the next group this thread reaches (G / 64 k-blocks on, at least one): its
                // parameters are fetched now, a whole group ahead of their use
                const int gn = g_cur + (lg >= 6 ? 1 : (kGemmKB >> lg));
                if ((gn << lg) < K) {
                    sc_next = __ldg(srow + gn);
                    if (zp) zw_next = __ldg(zrow + (gn >> 3));
                }
            }
            ok = mbar_wait(&wfull[s], (j / C::kWStages) & 1);
            if (ok && kb >= C::kABufs) ok = mbar_wait(&aempty[a], ((kb / C::kABufs) - 1) & 1);
            if (!ok) break;
            const uint4 packed = *reinterpret_cast<const uint4*>(
                smem + C::kWOff + s * C::kWBytes + wstage_swizzle<C::kWKB>(row * (32 * C::kWKB) + sb * 32 + kh * 16));
            uint4 v[4];
            v[0] = live ? dequant_word(packed.x, zmagic, zneg16, s2) : make_uint4(0, 0, 0, 0);
            v[1] = live ? dequant_word(packed.y, zmagic, zneg16, s2) : make_uint4(0, 0, 0, 0);
            v[2] = live ? dequant_word(packed.z, zmagic, zneg16, s2) : make_uint4(0, 0, 0, 0);
            v[3] = live ? dequant_word(packed.w, zmagic, zneg16, s2) : make_uint4(0, 0, 0, 0);
            __syncwarp();
            if (lane == 0 && (sb == C::kWKB - 1 || kb == num_kb - 1))
                mbar_arrive(&wempty[s]);                // the stage's packed words are in registers
            uint8_t* atile = smem + C::kAOff + a * C::kABytes + rt * C::kATileBytes;
#pragma unroll
            for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(atile + sw128_offset(r, kh * 4 + c)) = v[c];
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[a]);
        }
        if (ok && mbar_wait(tfull, 0)) {
            tc_fence_after();
            const int q = warp & 3;                        // TMEM lane quarter this warp may access
            const int set = (warp - 3) >> 2;               // 0..3: four warps per lane quarter
            const int ert = set >> 1;                      // accumulator (row tile) of this set
            const int t0 = (set & 1) * (kWideBN / 2);      // its 128 token columns
            const int nn = n0 + ert * kGemmTileN + q * 32 + lane;
            for (int c = 0; c < kWideBN / 2; c += 16) {
                uint32_t rv[16];
                tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ert * kWideBN + t0 + c), rv);
                tmem_ld_wait();
                if (nn < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + t0 + c + j;
                        if (m < M) Y[(size_t)m * N + nn] = f2h_rn(__uint_as_float(rv[j]));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Y = fp16(sum over the splits of the fp32 partial sums), the splits added in order.
__global__ void gemm_split_reduce_kernel(const float* __restrict__ part, int splits, size_t count,
                                         uint16_t* __restrict__ Y) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < count; i += (size_t)gridDim.x * blockDim.x) {
        float acc = part[i];
        for (int z = 1; z < splits; ++z) acc += part[(size_t)z * count + i];
        Y[i] = f2h_rn(acc);
    }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [rows][cols] of `esize`-byte elements; box [box_rows][box_cols].
inline bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int esize, uint64_t rows,
                         uint64_t cols, uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swz) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (uint64_t)esize};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D tensor with dims {d0 (innermost), d1, d2}, byte strides s1 (of d1) and s2 (of d2),
// box {b0, b1, b2}; no swizzle.
inline bool make_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
awq_status launch_gemm_bn(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                          const uint32_t* qzeros, int N, int K, int G, int zp, uint16_t* Y, cudaStream_t st,
                          int splits = 1, float* part = nullptr) {
    using C = GemmCfg<BN>;
    CUtensorMap tx, tq;
    if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)M, (uint64_t)K, BN, kGemmKB,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    if (!make_tmap_2d(&tq, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)N, (uint64_t)(K / 8), kGemmTileN,
                      C::kWKB * kGemmKB / 8, CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    auto kern = gemm_w4a16_kernel<BN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return AWQ_ERR_CUDA;
    const int num_kb = ceil_div(K, kGemmKB);
    if (splits < 1 || part == nullptr) splits = 1;
    // each split a whole number of packed-weight stages
    const int kb_per = ceil_div(ceil_div(num_kb, splits), C::kWKB) * C::kWKB;
    splits = ceil_div(num_kb, kb_per);
    dim3 grid(ceil_div(M, BN), ceil_div(N, kGemmTileN), splits);
    if (grid.y > 65535u) return AWQ_ERR_UNSUPPORTED;
    kern<<<grid, kGemmThreads, C::kSmemBytes, st>>>(tx, tq, scales, qzeros, M, N, K, G, zp, Y, kb_per,
                                                    splits > 1 ? part : nullptr);
    if (splits > 1) {
        const size_t count = (size_t)M * N;
        const unsigned blocks = (unsigned)std::min<size_t>((count + 255) / 256, 4096);
        gemm_split_reduce_kernel<<<blocks, 256, 0, st>>>(part, splits, count, Y);
    }
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// K splits of the 128-channel form for a batch whose tiles leave SMs idle (one CTA per
// SM).  Model of a split's time: a fixed start (TMA round trips, TMEM, the epilogue;
// about 3000 cycles) plus its k-blocks (about 400 cycles each with batched
// dequantisation), times the waves the CTAs take; the split count minimising it, each
// split at least 4 k-blocks, at most 16 splits.  1 = none.
inline int gemm_splits(int M, int N, int K, int sms) {
    const int bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    const long long tiles = (long long)ceil_div(M, bn) * ceil_div(N, kGemmTileN);
    const int num_kb = ceil_div(K, kGemmKB);
    if (tiles >= sms) return 1;
    int best = 1;
    double best_t = 1e300;
    for (int s = 1; s <= 16 && s <= std::max(1, num_kb / 4); ++s) {
        const double waves = (double)((tiles * s + sms - 1) / sms);
        const double t = waves * (3000.0 + 400.0 * ceil_div(num_kb, s));
        if (t < best_t * 0.999) best_t = t, best = s;
    }
    return best;
}

// Workspace of the GEMM: the fp32 partial sums of the split-K form (0 when it is not used).
inline size_t gemm_workspace_bytes(int M, int N, int K, int sms) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    const int s = gemm_splits(M, N, K, sms);
    return s > 1 ? (size_t)s * M * N * 4 : 0;
}

inline awq_status launch_gemm_wide(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                                   const uint32_t* qzeros, int N, int K, int G, int zp, uint16_t* Y, cudaStream_t st) {
    using C = GemmWideCfg;
    CUtensorMap tx, tq;
    if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)M, (uint64_t)K, kWideBN, kGemmKB,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    constexpr CUtensorMapSwizzle wswz = C::kWKB == 4   ? CU_TENSOR_MAP_SWIZZLE_128B
                                        : C::kWKB == 2 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                       : CU_TENSOR_MAP_SWIZZLE_NONE;
    if (!make_tmap_2d(&tq, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)N, (uint64_t)(K / 8), kWideRows,
                      C::kWKB * kGemmKB / 8, wswz))
        return AWQ_ERR_CUDA;
    if (cudaFuncSetAttribute(gemm_w4a16_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
        return AWQ_ERR_CUDA;
    dim3 grid(ceil_div(M, kWideBN), ceil_div(N, kWideRows));
    if (grid.y > 65535u) return AWQ_ERR_UNSUPPORTED;
    gemm_w4a16_wide_kernel<<<grid, kWideThreads, C::kSmemBytes, st>>>(tx, tq, scales, qzeros, M, N, K, G, zp, Y);
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// The wide form does twice the work per tile and, by the k-block rate of the two forms,
// about kWideGain times the work per unit time; it is used where that beats the wave
// count of the 128-channel form (one resident CTA per SM for both).
constexpr double kWideGain = 1.6;

inline bool use_wide_gemm(int M, int N, int sms) {
    if (M <= 128) return false;
    const long long mt = ceil_div(M, kWideBN);
    const long long narrow = mt * ceil_div(N, kGemmTileN), wide = mt * ceil_div(N, kWideRows);
    const double t_narrow = (double)((narrow + sms - 1) / sms);
    const double t_wide = (double)((wide + sms - 1) / sms) * 2.0 / kWideGain;
    return t_wide < t_narrow;
}

inline awq_status launch_gemm_w4a16(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                                    const uint32_t* qzeros, int N, int K, int G, int zp, uint16_t* Y, cudaStream_t st,
                                    int sms, void* ws, size_t ws_bytes) {
    if (use_wide_gemm(M, N, sms)) return launch_gemm_wide(X, M, qweight, scales, qzeros, N, K, G, zp, Y, st);
    // split K over the caller's workspace when the tiles alone leave SMs idle (as many
    // splits as the workspace holds, up to the chosen number)
    int splits = gemm_splits(M, N, K, sms);
    if (splits > 1) {
        const size_t per = (size_t)M * N * 4;
        const size_t fit = (ws && per) ? ws_bytes / per : 0;
        splits = (int)std::min<size_t>((size_t)splits, fit);
    }
    float* part = splits > 1 ? static_cast<float*>(ws) : nullptr;
#define AWQ_GEMM_BN(BB) return launch_gemm_bn<BB>(X, M, qweight, scales, qzeros, N, K, G, zp, Y, st, splits, part)
    if (M <= 16) AWQ_GEMM_BN(16);
    if (M <= 32) AWQ_GEMM_BN(32);
    if (M <= 64) AWQ_GEMM_BN(64);
    if (M <= 128) AWQ_GEMM_BN(128);
    AWQ_GEMM_BN(256);
#undef AWQ_GEMM_BN
}

}  // namespace awq
