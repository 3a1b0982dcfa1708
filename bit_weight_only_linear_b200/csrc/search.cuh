// Activation-aware scale search on the sm_100a tensor cores.
//
// Source: "AI-Research-SKILLs AWQ advanced usage guide" (lshu.cn), section 算法原理:
// choose the per-input-channel scale s that minimises L(s) = || Q(W s)(s^-1 X) - W X ||,
// with s derived from the activation distribution; the search space is
// s = mean|X|^alpha over a grid of alpha.  Per alpha (all fp32 steps as in
// awq_quantize_pack, the rest in fp64):
//   m_k    = mean_t |X[t][k]|                       (exact: fp64 sums of fp16 values)
//   s_k    = fp16(max(pow(m_k, alpha), 2^-14))
//   dW     = (Q(W s) - W s) / s  = Q(W s)/s - W      (difference exact in fp64, quotient
//                                                      in fp32: within one fp32 ulp)
//   loss   = mean_{t,n} (sum_k X[t][k] dW[n][k])^2
// The loss GEMM E = X dW^T is a dense contraction and runs on tcgen05: dW of each
// row n is scaled by 2^e_n (its largest entry lands in [2^13, 2^14)) and split into
// two fp16 terms hi + lo (a 22-bit significand), so E = X hi^T + X lo^T is two MMAs
// into one fp32 TMEM accumulator with exact products; the epilogue undoes 2^e_n per
// column and sums E^2 in fp64.  E never leaves the SM.  Partial sums per tile are
// added in a fixed order, so the loss is deterministic.
#pragma once

#include "common.cuh"
#include "gemm_sm100.cuh"
#include "quantize.cuh"
#include "sm100.cuh"

namespace awq {

constexpr int kSearchMaxGrid = 64;     // n_grid upper bound (s table and losses)
constexpr int kSearchBatch = 8;        // alphas evaluated per pass
constexpr int kSearchTileM = 128;      // calibration tokens per tile (MMA M)
constexpr int kSearchTileN = 128;      // output channels per tile (MMA N)
constexpr int kSearchStages = 4;
constexpr int kSearchThreads = 192;    // TMA warp, MMA warp, 4 epilogue warps

struct SearchWorkspace {
    double* colsum;      // [K]
    uint16_t* s_all;     // [kSearchMaxGrid][K]
    uint16_t* dw;        // [kSearchBatch][N][2*Kp], Kp = K rounded up to 64: per 64-channel block, 64 hi then 64 lo
    int32_t* row_exp;    // [kSearchBatch][N]
    double* partial;     // [kSearchBatch][tiles]
    double* losses;      // [kSearchMaxGrid]
    size_t bytes;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// K rounded up to whole 64-channel blocks (the dW row pitch is 2 * Kp).
__host__ __device__ inline int search_kp(int K) { return (K + 63) & ~63; }

inline SearchWorkspace search_layout(void* base, int M, int N, int K) {
    SearchWorkspace w;
    size_t off = 0;
    char* b = static_cast<char*>(base);
    auto take = [&](size_t bytes) {
        char* p = b ? b + off : nullptr;
        off += align256(bytes);
        return p;
    };
    const size_t tiles = (size_t)ceil_div(M, kSearchTileM) * ceil_div(N, kSearchTileN);
    w.colsum = reinterpret_cast<double*>(take((size_t)K * 8));
    w.s_all = reinterpret_cast<uint16_t*>(take((size_t)kSearchMaxGrid * K * 2));
    w.dw = reinterpret_cast<uint16_t*>(take((size_t)kSearchBatch * N * 2 * search_kp(K) * 2));
    w.row_exp = reinterpret_cast<int32_t*>(take((size_t)kSearchBatch * N * 4));
    w.partial = reinterpret_cast<double*>(take((size_t)kSearchBatch * tiles * 8));
    w.losses = reinterpret_cast<double*>(take((size_t)kSearchMaxGrid * 8));
    w.bytes = off;
    return w;
}

inline size_t search_workspace_bytes(int M, int N, int K, int /*G*/, int /*n_grid*/) {
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return search_layout(nullptr, M, N, K).bytes;
}

// ---------------------------------------------------------------------------
// dW = Q(W s)/s - W for one (alpha, row): block of 256 threads, 8 channels each per
// 2048-channel chunk (the group reduction is the one of quantize_pack_kernel).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kQuantThreads)
search_delta_kernel(const uint16_t* __restrict__ W, const uint16_t* __restrict__ s_batch, int N, int K, int G,
                    int zero_point, uint16_t* __restrict__ dw, int32_t* __restrict__ row_exp) {
    extern __shared__ float dsm[];   // [K] dW of this row, then [32] block-max scratch
    const int row = blockIdx.x;
    const int a = blockIdx.y;
    const uint16_t* s = s_batch + (size_t)a * K;
    const bool zp = zero_point != 0;
    float amax = 0.0f;
    for (int c0 = 0; c0 < K; c0 += kQuantChunk) {
        const int k0 = c0 + threadIdx.x * 8;
        const bool active = k0 < K;
        float ws[8], sv[8];
        if (active) {
            const uint4 wv = *reinterpret_cast<const uint4*>(W + (size_t)row * K + k0);
            const uint4 svv = *reinterpret_cast<const uint4*>(s + k0);
            const uint16_t* wh = reinterpret_cast<const uint16_t*>(&wv);
            const uint16_t* sh = reinterpret_cast<const uint16_t*>(&svv);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                sv[i] = h2f(sh[i]);
                ws[i] = __fmul_rn(h2f(wh[i]), sv[i]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) ws[i] = 0.0f, sv[i] = 1.0f;
        }
        float mx = ws[0], mn = ws[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            mx = fmaxf(mx, ws[i]);
            mn = fminf(mn, ws[i]);
        }
        seg_minmax(mx, mn, G >> 3);
        const GroupParams p = group_params(mx, mn, zp);
        if (active) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float q = (float)quant_code(ws[i], p, zp);
                const float deq = __fmul_rn(q - p.zero, p.sc);                        // exact
                // fp32 quotient of the fp64-exact difference: within one fp32 ulp of the
                // correctly rounded dW, far below the 22-bit hi/lo split that follows
                const float df = __fdiv_rn((float)((double)deq - (double)ws[i]), sv[i]);
                dsm[k0 + i] = df;
                amax = fmaxf(amax, fabsf(df));
            }
        }
    }
    // block max of |dW|
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    float* red = dsm + K;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (kQuantThreads / 32) ? red[threadIdx.x] : 0.0f;
        for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const float rmax = red[0];
    int e = 0;
    if (rmax > 0.0f) {
        int ex;
        frexpf(rmax, &ex);            // rmax = f 2^ex, f in [0.5, 1)
        e = 14 - ex;                  // rmax 2^e in [2^13, 2^14)
    }
    if (threadIdx.x == 0) row_exp[(size_t)a * N + row] = e;
    // hi/lo split, written as [64 hi | 64 lo] per 64-channel block; the tail of the
    // last block (k >= K) is written as zeros
    const int kp = search_kp(K);
    uint16_t* out = dw + ((size_t)a * N + row) * (size_t)(2 * kp);
    for (int k0 = threadIdx.x * 8; k0 < kp; k0 += kQuantThreads * 8) {   // 8 channels, 16-byte stores
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            uint16_t h2[2], l2[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int k = k0 + i + j;
                const float v = k < K ? ldexpf(dsm[k], e) : 0.0f;
                h2[j] = f2h_rn(v);
                l2[j] = f2h_rn(v - h2f(h2[j]));   // exact difference
            }
            hw[i / 2] = (uint32_t)h2[0] | ((uint32_t)h2[1] << 16);
            lw[i / 2] = (uint32_t)l2[0] | ((uint32_t)l2[1] << 16);
        }
        const int kb = k0 >> 6, w = k0 & 63;
        *reinterpret_cast<uint4*>(out + kb * 128 + w) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(out + kb * 128 + 64 + w) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
}

// ---------------------------------------------------------------------------
// Sum of squares of E = X dW^T for one alpha (blockIdx.z), one 128 x 128 tile.
// ---------------------------------------------------------------------------
struct SearchGemmCfg {
    static constexpr int kABytes = kSearchTileM * 128;   // X tile: 128 rows x 64 fp16
    static constexpr int kBBytes = kSearchTileN * 128;   // one dW term tile
    static constexpr int kStageBytes = kABytes + 2 * kBBytes;
    static constexpr int kBarOff = kSearchStages * kStageBytes;
    static constexpr int kNumBars = 2 * kSearchStages + 1;
    static constexpr int kExpOff = kBarOff + kNumBars * 8;          // [kSearchTileN] int
    static constexpr int kRedOff = kExpOff + kSearchTileN * 4;      // [4] double
    static constexpr int kTmemPtrOff = kRedOff + 4 * 8;
    static constexpr int kSmemBytes = kTmemPtrOff + 16 + 1024;
};

__global__ void __launch_bounds__(kSearchThreads, 1)
search_sumsq_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_dw, int M,
                    int N, int K, const int32_t* __restrict__ row_exp, double* __restrict__ partial) {
    using C = SearchGemmCfg;
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
    uint64_t* empty = full + kSearchStages;
    uint64_t* tfull = empty + kSearchStages;
    int32_t* exps = reinterpret_cast<int32_t*>(smem + C::kExpOff);
    double* red = reinterpret_cast<double*>(smem + C::kRedOff);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::kTmemPtrOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kSearchTileM;
    const int n0 = blockIdx.y * kSearchTileN;
    const int a = blockIdx.z;
    const int num_kb = ceil_div(K, 64);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSearchStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_fence_init();
        prefetch_tensormap(&tmap_x);
        prefetch_tensormap(&tmap_dw);
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, kSearchTileN);
        tmem_relinquish();
    }
    for (int j = threadIdx.x; j < kSearchTileN; j += kSearchThreads)
        exps[j] = (n0 + j < N) ? row_exp[(size_t)a * N + n0 + j] : 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0) {
        if (lane == 0) {
            int issued = 0;
            const int brow = a * N + n0;     // row of the [batch*N][2K] view
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % kSearchStages;
                if (kb >= kSearchStages && !mbar_wait(&empty[s], ((kb / kSearchStages) - 1) & 1)) break;
                uint8_t* st = smem + s * C::kStageBytes;
                mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                tma_load_2d(st, &tmap_x, &full[s], kb * 64, m0);
                tma_load_2d(st + C::kABytes, &tmap_dw, &full[s], kb * 128, brow);
                tma_load_2d(st + C::kABytes + C::kBBytes, &tmap_dw, &full[s], kb * 128 + 64, brow);
                ++issued;
            }
            for (int kb = issued - 1; kb >= 0 && kb >= issued - kSearchStages; --kb)
                mbar_wait(&full[kb % kSearchStages], (kb / kSearchStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(kSearchTileM, kSearchTileN);
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb) {
                const int s = kb % kSearchStages;
                if (!mbar_wait(&full[s], (kb / kSearchStages) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * C::kStageBytes);
                const uint64_t ad = desc_sw128_kmajor(st);
                const uint64_t bh = desc_sw128_kmajor(st + C::kABytes);
                const uint64_t bl = desc_sw128_kmajor(st + C::kABytes + C::kBBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_f16(tmem, ad + 2 * kk, bh + 2 * kk, idesc, (kb | kk) != 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_f16(tmem, ad + 2 * kk, bl + 2 * kk, idesc, 1u);
                mma_commit(&empty[s]);
            }
            mma_commit(tfull);
            if (!ok) mbar_wait(tfull, 0);
        }
    } else {
        // epilogue: warps 2..5, TMEM lane quarter = warp % 4
        const int q = warp & 3;
        double acc = 0.0;
        if (mbar_wait(tfull, 0)) {
            tc_fence_after();
            const int m = m0 + q * 32 + lane;
            for (int c = 0; c < kSearchTileN; c += 16) {
                uint32_t r[16];
                tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, r);
                tmem_ld_wait();
                if (m < M) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (n0 + c + j < N) {
                            const double e = ldexp((double)__uint_as_float(r[j]), -exps[c + j]);
                            acc = fma(e, e, acc);
                        }
                    }
                }
            }
        }
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) red[q] = acc;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kSearchTileN);
    }
    if (threadIdx.x == 0) {
        const size_t tiles = (size_t)gridDim.x * gridDim.y;
        partial[(size_t)a * tiles + (size_t)blockIdx.y * gridDim.x + blockIdx.x] = ((red[0] + red[1]) + red[2]) + red[3];
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

inline awq_status run_scale_search(const uint16_t* X, int M, const uint16_t* W, int N, int K, int G, int zp,
                                   int n_grid, uint16_t* s_out, double* losses_out, int32_t* best_out, void* ws,
                                   cudaStream_t st, int sms) {
    (void)sms;
    const SearchWorkspace w = search_layout(ws, M, N, K);
    if (cudaMemsetAsync(w.colsum, 0, (size_t)K * 8, st) != cudaSuccess) return AWQ_ERR_CUDA;
    {
        dim3 grid(ceil_div(K / 8, 128), (unsigned)min(M, 64));
        abs_colsum_kernel<<<grid, 128, 0, st>>>(X, M, K, w.colsum);
    }
    {
        dim3 grid(ceil_div(K, 256), n_grid);
        scales_for_alphas_kernel<<<grid, 256, 0, st>>>(w.colsum, M, K, n_grid, w.s_all);
    }
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;

    const size_t dsm = (size_t)K * 4 + 32 * 4;
    if (dsm > 48 * 1024 &&
        cudaFuncSetAttribute(search_delta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm) != cudaSuccess)
        return AWQ_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(search_sumsq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SearchGemmCfg::kSmemBytes) != cudaSuccess)
        return AWQ_ERR_CUDA;
    CUtensorMap tx;
    if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)M, (uint64_t)K, kSearchTileM, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    const int mt = ceil_div(M, kSearchTileM), nt = ceil_div(N, kSearchTileN);
    for (int b0 = 0; b0 < n_grid; b0 += kSearchBatch) {
        const int na = min(kSearchBatch, n_grid - b0);
        search_delta_kernel<<<dim3(N, na), kQuantThreads, dsm, st>>>(W, w.s_all + (size_t)b0 * K, N, K, G, zp, w.dw,
                                                                     w.row_exp);
        CUtensorMap td;
        if (!make_tmap_2d(&td, w.dw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)na * N, (uint64_t)2 * search_kp(K),
                          kSearchTileN, 64, CU_TENSOR_MAP_SWIZZLE_128B))
            return AWQ_ERR_CUDA;
        search_sumsq_kernel<<<dim3(mt, nt, na), kSearchThreads, SearchGemmCfg::kSmemBytes, st>>>(
            tx, td, M, N, K, w.row_exp, w.partial);
        search_loss_kernel<<<na, 256, 0, st>>>(w.partial, mt * nt, 1.0 / ((double)M * (double)N), w.losses + b0);
        if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
    }
    search_select_kernel<<<ceil_div(K, 256), 256, 0, st>>>(w.losses, n_grid, w.s_all, K, s_out, best_out, losses_out);
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Same search over caller-provided scratch of bounded size: one alpha and one
// chunk of output channels at a time, the chunk's tile sums added to the running
// loss in a fixed order (deterministic).  Used by awq_scale_search_noalloc.
// ---------------------------------------------------------------------------

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

struct ChunkedSearchLayout {
    double* colsum;      // [K]
    uint16_t* s_all;     // [kSearchMaxGrid][K]
    double* losses;      // [kSearchMaxGrid]
    double* partial;     // [partial_cap]
    int32_t* row_exp;    // [nc]
    uint16_t* dw;        // [nc][2*Kp]
    int nc;              // output channels per chunk (multiple of kSearchTileN), 0 if it does not fit
    size_t partial_cap;
};

inline ChunkedSearchLayout chunked_search_layout(void* base, size_t bytes, int M, int N, int K) {
    ChunkedSearchLayout L = {};
    char* b = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t n) {
        char* p = b + off;
        off += align256(n);
        return p;
    };
    L.colsum = reinterpret_cast<double*>(take((size_t)K * 8));
    L.s_all = reinterpret_cast<uint16_t*>(take((size_t)kSearchMaxGrid * K * 2));
    L.losses = reinterpret_cast<double*>(take((size_t)kSearchMaxGrid * 8));
    L.partial_cap = 32768;   // doubles
    L.partial = reinterpret_cast<double*>(take(L.partial_cap * 8));
    if (off >= bytes) return L;
    const size_t per_row = (size_t)2 * search_kp(K) * 2 + 4;      // dW row + its exponent
    size_t nc = (bytes - off - 512) / per_row;
    nc = nc / kSearchTileN * kSearchTileN;
    const size_t n_cap = (size_t)ceil_div(N, kSearchTileN) * kSearchTileN;
    if (nc > n_cap) nc = n_cap;
    const size_t mt = (size_t)ceil_div(M, kSearchTileM);
    while (nc > 0 && mt * (nc / kSearchTileN) > L.partial_cap) nc -= kSearchTileN;
    L.nc = (int)nc;
    if (nc == 0) return L;
    L.row_exp = reinterpret_cast<int32_t*>(take(nc * 4));
    L.dw = reinterpret_cast<uint16_t*>(take(nc * 2 * (size_t)search_kp(K) * 2));
    if (off > bytes) L.nc = 0;
    return L;
}

inline awq_status run_scale_search_chunked(const uint16_t* X, int M, const uint16_t* W, int N, int K, int G, int zp,
                                           int n_grid, uint16_t* s_out, double* losses_out, int32_t* best_out,
                                           const ChunkedSearchLayout& L, cudaStream_t st) {
    if (L.nc <= 0) return AWQ_ERR_UNSUPPORTED;
    if (cudaMemsetAsync(L.colsum, 0, (size_t)K * 8, st) != cudaSuccess) return AWQ_ERR_CUDA;
    abs_colsum_kernel<<<dim3(ceil_div(K / 8, 128), (unsigned)min(M, 64)), 128, 0, st>>>(X, M, K, L.colsum);
    scales_for_alphas_kernel<<<dim3(ceil_div(K, 256), n_grid), 256, 0, st>>>(L.colsum, M, K, n_grid, L.s_all);
    if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
    const size_t dsm = (size_t)K * 4 + 32 * 4;
    if (dsm > 48 * 1024 &&
        cudaFuncSetAttribute(search_delta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsm) != cudaSuccess)
        return AWQ_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(search_sumsq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SearchGemmCfg::kSmemBytes) != cudaSuccess)
        return AWQ_ERR_CUDA;
    CUtensorMap tx;
    if (!make_tmap_2d(&tx, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)M, (uint64_t)K, kSearchTileM, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return AWQ_ERR_CUDA;
    const int mt = ceil_div(M, kSearchTileM);
    const double inv_mn = 1.0 / ((double)M * (double)N);
    for (int a = 0; a < n_grid; ++a) {
        for (int n0 = 0; n0 < N; n0 += L.nc) {
            const int nc = min(L.nc, N - n0);
            search_delta_kernel<<<dim3(nc, 1), kQuantThreads, dsm, st>>>(W + (size_t)n0 * K, L.s_all + (size_t)a * K,
                                                                        nc, K, G, zp, L.dw, L.row_exp);
            CUtensorMap td;
            if (!make_tmap_2d(&td, L.dw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)nc, (uint64_t)2 * search_kp(K),
                              kSearchTileN, 64, CU_TENSOR_MAP_SWIZZLE_128B))
                return AWQ_ERR_CUDA;
            const int ntc = ceil_div(nc, kSearchTileN);
            search_sumsq_kernel<<<dim3(mt, ntc, 1), kSearchThreads, SearchGemmCfg::kSmemBytes, st>>>(
                tx, td, M, nc, K, L.row_exp, L.partial);
            search_accum_kernel<<<1, 256, 0, st>>>(L.partial, mt * ntc, n0 == 0, n0 + nc >= N, inv_mn, L.losses + a);
            if (cudaGetLastError() != cudaSuccess) return AWQ_ERR_CUDA;
        }
    }
    search_select_kernel<<<ceil_div(K, 256), 256, 0, st>>>(L.losses, n_grid, L.s_all, K, s_out, best_out, losses_out);
    return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
