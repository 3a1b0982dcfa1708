// Host side of the decode GEMV: device facts, the choice between the TMA-staged and
// the register-ring kernel with its stages, parameter slots and grid (a launch plan,
// cached per device and (M, N, K, G)), the cached TMA view of each weight matrix, and
// the launch itself.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "common.cuh"
#include "gemm_sm100.cuh"
#include "gemv.cuh"
#include "launch.cuh"

namespace awq {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int max_smem_optin = 0;
    int smem_per_sm = 0;
};

inline std::mutex g_mu;                 // guards every per-device cache of the library
inline DeviceInfo g_dev[kMaxDevices];

inline bool device_info(DeviceInfo& out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
            return false;
        if (cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
            return false;
        d.ready = true;
    }
    out = d;
    return true;
}

// Stages and raw parameter slots of the TMA GEMV.  Parameters are small (1/32 of the
// weight bytes at G = 128), so every row group a CTA will take gets a raw slot when
// that fits (up to 8): all parameter copies are then issued at the start and none
// waits behind the weight stream.  Preference: two CTAs per SM, then at least four
// stages, then the most parameter slots, then the deepest ring (3..6 stages); false
// if nothing fits.
inline bool pick_gemv_tma(const DeviceInfo& d, int M, int N, int K, int G, int& S, int& PR, int& ctas) {
    const int n_rg = N / kGemvRows;
    for (ctas = 2; ctas >= 1; --ctas) {
        const int slots = d.sms * ctas;
        const int grid = n_rg < slots ? n_rg : slots;
        const int per_cta = (n_rg + grid - 1) / grid;
        const int pr_max = per_cta < kTmaMaxParamSlots ? (per_cta > 2 ? per_cta : 2) : kTmaMaxParamSlots;
        for (int s_floor = kTmaMinStages + 1; s_floor >= kTmaMinStages; --s_floor)
            for (PR = pr_max; PR >= 2; --PR)
                for (S = kTmaMaxStages; S >= s_floor; --S) {
                    const size_t b = GemvTmaSmem(M, K, G, S, PR).bytes();
                    if (b <= (size_t)d.max_smem_optin && (size_t)ctas * (b + 1024) <= (size_t)d.smem_per_sm)
                        return true;
                }
    }
    return false;
}

// ---------------------------------------------------------------------------
// GEMV launch plans.  Everything a launch needs that depends only on the device and
// on (M, N, K, G) -- which kernel, its stages and parameter slots, grid and shared
// memory -- is worked out on the first call and cached, and so is the TMA view of
// each weight matrix (per device, qweight pointer, N and K).  A later call makes one
// lookup under one lock, then the launch.
// ---------------------------------------------------------------------------
struct GemvPlan {
    int dev, M, N, K, G;
    bool tma;          // TMA-staged kernel, else the register-ring kernel
    const void* fn;
    int grid, S, PR, ks;
    size_t smem;
};

struct GemvTmap {
    int dev;
    const void* base;
    int N, K;
    CUtensorMap map;
};

constexpr int kGemvTmapCache = 256;
inline std::vector<GemvPlan> g_gemv_plans;
inline GemvTmap g_gemv_tmaps[kGemvTmapCache];
inline int g_gemv_tmap_count = 0, g_gemv_tmap_next = 0;

inline const void* gemv_tma_fn(int G, bool one) {
    switch (G) {
        case 32: return one ? (const void*)gemv_tma_kernel<32, true> : (const void*)gemv_tma_kernel<32, false>;
        case 64: return one ? (const void*)gemv_tma_kernel<64, true> : (const void*)gemv_tma_kernel<64, false>;
        case 128: return one ? (const void*)gemv_tma_kernel<128, true> : (const void*)gemv_tma_kernel<128, false>;
        default: return one ? (const void*)gemv_tma_kernel<256, true> : (const void*)gemv_tma_kernel<256, false>;
    }
}

inline const void* gemv_mma_fn(int WT, bool one) {
    switch (WT) {
        case 1: return one ? (const void*)gemv_mma_kernel<1, true> : (const void*)gemv_mma_kernel<1, false>;
        case 2: return one ? (const void*)gemv_mma_kernel<2, true> : (const void*)gemv_mma_kernel<2, false>;
        default: return one ? (const void*)gemv_mma_kernel<4, true> : (const void*)gemv_mma_kernel<4, false>;
    }
}

// Fills p (keyed fields set by the caller).  The TMA kernel takes every shape with whole
// 16-row groups and whole 128-code blocks whose staging fits; the register-ring kernel
// takes the rest.
inline awq_status build_gemv_plan(GemvPlan& p, const DeviceInfo& d) {
    int S = 0, PR = 0, ctas = 0;
    if (p.N % kGemvRows == 0 && p.K % 128 == 0 && pick_gemv_tma(d, p.M, p.N, p.K, p.G, S, PR, ctas)) {
        p.tma = true;
        p.fn = gemv_tma_fn(p.G, p.M == 1);
        p.S = S;
        p.PR = PR;
        p.ks = 0;
        p.smem = GemvTmaSmem(p.M, p.K, p.G, S, PR).bytes();
        int occ = 0;
        if (!kernel_occupancy(p.fn, kTmaThreads, p.smem, occ) || occ < 1) return AWQ_ERR_CUDA;
        // one CTA per resident slot, row groups dealt round-robin
        const int n_rg = p.N / kGemvRows;
        const int slots = d.sms * occ;
        p.grid = n_rg < slots ? n_rg : slots;
        return AWQ_OK;
    }
    p.tma = false;
    const int WT = gemv_words_per_thread(p.G);
    p.fn = gemv_mma_fn(WT, p.M == 1);
    const int nsteps = p.K / (32 * WT);
    p.smem = GemvSmem::bytes(p.M, p.K, nsteps);
    if (p.smem > (size_t)d.max_smem_optin) return AWQ_ERR_UNSUPPORTED;
    int occ = 0;
    if (!kernel_occupancy(p.fn, kGemvThreads, p.smem, occ) || occ < 1) return AWQ_ERR_CUDA;
    // persistent grid: at most one wave, row-group iterations spread evenly over the CTAs
    const int UK = kGemvUnitWords / WT;
    const int units = ceil_div(nsteps, UK);
    const int slots = d.sms * occ;
    p.ks = gemv_ks(units, ceil_div(p.N, kGemvRows), slots);
    const int rpi = kGemvWarps / p.ks;
    const int n_it = ceil_div(ceil_div(p.N, kGemvRows), rpi);
    const int per_cta = ceil_div(n_it, slots);
    p.grid = ceil_div(n_it, per_cta);
    p.S = p.PR = 0;
    return AWQ_OK;
}

// The cached plan for (current device, M, N, K, G) and, for the TMA kernel, the cached
// view of qweight.
inline awq_status gemv_plan(const uint32_t* qweight, int M, int N, int K, int G, GemvPlan& out, CUtensorMap& tq) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
    DeviceInfo d;                          // (takes g_mu itself: look it up before locking)
    if (!device_info(d)) return AWQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    const GemvPlan* found = nullptr;
    for (const GemvPlan& p : g_gemv_plans)
        if (p.dev == dev && p.M == M && p.N == N && p.K == K && p.G == G) {
            found = &p;
            break;
        }
    if (!found) {
        GemvPlan p = {};
        p.dev = dev, p.M = M, p.N = N, p.K = K, p.G = G;
        const awq_status st = build_gemv_plan(p, d);
        if (st != AWQ_OK) return st;
        g_gemv_plans.push_back(p);
        found = &g_gemv_plans.back();
    }
    out = *found;
    if (!out.tma) return AWQ_OK;
    for (int i = 0; i < g_gemv_tmap_count; ++i) {
        const GemvTmap& e = g_gemv_tmaps[i];
        if (e.dev == dev && e.base == qweight && e.N == N && e.K == K) {
            tq = e.map;
            return AWQ_OK;
        }
    }
    // qweight [N][K/8] words viewed as {16 words, N rows, K/128 blocks}
    if (!make_tmap_3d(&tq, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT32, 16, (uint64_t)N, (uint64_t)(K / 128),
                      (uint64_t)K / 2, 64, 16, kGemvRows, kTmaKC / 128))
        return AWQ_ERR_CUDA;
    const int slot = g_gemv_tmap_count < kGemvTmapCache ? g_gemv_tmap_count++ : (g_gemv_tmap_next++ % kGemvTmapCache);
    g_gemv_tmaps[slot] = {dev, qweight, N, K, tq};
    return AWQ_OK;
}

inline awq_status launch_gemv(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                       const uint32_t* qzeros, int N, int K, const awq_quant_config& cfg, uint16_t* Y,
                       cudaStream_t st) {
    GemvPlan p;
    CUtensorMap tq;
    const awq_status ps = gemv_plan(qweight, M, N, K, cfg.q_group_size, p, tq);
    if (ps == AWQ_ERR_UNSUPPORTED && M > 1) {
        // the M rows of X are staged in shared memory: when they do not fit (long rows,
        // e.g. 8 x 14336), the batch is split and each part is its own launch
        const int m1 = M / 2;
        const awq_status a = launch_gemv(X, m1, qweight, scales, qzeros, N, K, cfg, Y, st);
        if (a != AWQ_OK) return a;
        return launch_gemv(X + (size_t)m1 * K, M - m1, qweight, scales, qzeros, N, K, cfg, Y + (size_t)m1 * N, st);
    }
    if (ps != AWQ_OK) return ps;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(p.grid);
    lc.blockDim = dim3(p.tma ? kTmaThreads : kGemvThreads);
    lc.dynamicSmemBytes = p.smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int zp = cfg.zero_point, G = cfg.q_group_size;
    cudaError_t e;
    if (p.tma) {
        // (tmap_q, X, M, scales, qzeros, N, K, zero_point, Y, S, PR)
        void* args[] = {&tq, &X, &M, &scales, &qzeros, &N, &K, &zp, &Y, &p.S, &p.PR};
        e = cudaLaunchKernelExC(&lc, p.fn, args);
    } else {
        // (X, M, qweight, scales, qzeros, N, K, G, zero_point, ks, Y)
        void* args[] = {&X, &M, &qweight, &scales, &qzeros, &N, &K, &G, &zp, &p.ks, &Y};
        e = cudaLaunchKernelExC(&lc, p.fn, args);
    }
    return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

}  // namespace awq
