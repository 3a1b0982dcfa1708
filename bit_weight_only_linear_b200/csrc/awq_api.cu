// C ABI of the AWQ W4A16 library: argument checks, launch configuration, and the
// entry points declared in include/awq.h.  The whole library is one translation
// unit (this file includes the kernel headers), so the device error word and the
// kernels share one module.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "launch.cuh"
#include "gemv.cuh"
#include "quantize.cuh"
#include "gemm_sm100.cuh"
#include "search.cuh"

using namespace awq;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int max_smem_optin = 0;
    int smem_per_sm = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

bool device_info(DeviceInfo& out) {
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

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

awq_status check_config(const awq_quant_config& c) {
    if (c.zero_point != 0 && c.zero_point != 1) return AWQ_ERR_INVALID_ARG;
    if (c.w_bit != 4) return AWQ_ERR_UNSUPPORTED;
    if (c.q_group_size != 32 && c.q_group_size != 64 && c.q_group_size != 128 && c.q_group_size != 256)
        return AWQ_ERR_UNSUPPORTED;
    return AWQ_OK;
}

awq_status check_shape(int N, int K, const awq_quant_config& c) {
    if (N <= 0 || K <= 0) return AWQ_ERR_INVALID_ARG;
    if (K % c.q_group_size != 0) return AWQ_ERR_INVALID_ARG;
    return AWQ_OK;
}

awq_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// Checks shared by the two linear entry points.
awq_status check_linear(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                        const uint32_t* qzeros, int N, int K, const awq_quant_config& cfg,
                        const uint16_t* Y) {
    awq_status st = check_config(cfg);
    if (st != AWQ_OK) return st;
    st = check_shape(N, K, cfg);
    if (st != AWQ_OK) return st;
    if (M <= 0) return AWQ_ERR_INVALID_ARG;
    if (!X || !qweight || !scales || !Y) return AWQ_ERR_INVALID_ARG;
    if (cfg.zero_point && !qzeros) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(qweight) || !aligned16(scales) || !aligned16(Y)) return AWQ_ERR_INVALID_ARG;
    if (qzeros && !aligned16(qzeros)) return AWQ_ERR_INVALID_ARG;
    return AWQ_OK;
}

// Stages and raw parameter slots of the TMA GEMV.  Parameters are small (1/32 of the
// weight bytes at G = 128), so every row group a CTA will take gets a raw slot when
// that fits (up to 8): all parameter copies are then issued at the start and none
// waits behind the weight stream.  Preference: two CTAs per SM, then at least four
// stages, then the most parameter slots, then the deepest ring (3..6 stages); false
// if nothing fits.
bool pick_gemv_tma(const DeviceInfo& d, int M, int N, int K, int G, int& S, int& PR, int& ctas) {
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
std::vector<GemvPlan> g_gemv_plans;
GemvTmap g_gemv_tmaps[kGemvTmapCache];
int g_gemv_tmap_count = 0, g_gemv_tmap_next = 0;

const void* gemv_tma_fn(int G, bool one) {
    switch (G) {
        case 32: return one ? (const void*)gemv_tma_kernel<32, true> : (const void*)gemv_tma_kernel<32, false>;
        case 64: return one ? (const void*)gemv_tma_kernel<64, true> : (const void*)gemv_tma_kernel<64, false>;
        case 128: return one ? (const void*)gemv_tma_kernel<128, true> : (const void*)gemv_tma_kernel<128, false>;
        default: return one ? (const void*)gemv_tma_kernel<256, true> : (const void*)gemv_tma_kernel<256, false>;
    }
}

const void* gemv_mma_fn(int WT, bool one) {
    switch (WT) {
        case 1: return one ? (const void*)gemv_mma_kernel<1, true> : (const void*)gemv_mma_kernel<1, false>;
        case 2: return one ? (const void*)gemv_mma_kernel<2, true> : (const void*)gemv_mma_kernel<2, false>;
        default: return one ? (const void*)gemv_mma_kernel<4, true> : (const void*)gemv_mma_kernel<4, false>;
    }
}

// Fills p (keyed fields set by the caller).  The TMA kernel takes every shape with whole
// 16-row groups and whole 128-code blocks whose staging fits; the register-ring kernel
// takes the rest.
awq_status build_gemv_plan(GemvPlan& p) {
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
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
awq_status gemv_plan(const uint32_t* qweight, int M, int N, int K, int G, GemvPlan& out, CUtensorMap& tq) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
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
        const awq_status st = build_gemv_plan(p);
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

awq_status launch_gemv(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                       const uint32_t* qzeros, int N, int K, const awq_quant_config& cfg, uint16_t* Y,
                       cudaStream_t st) {
    GemvPlan p;
    CUtensorMap tq;
    const awq_status ps = gemv_plan(qweight, M, N, K, cfg.q_group_size, p, tq);
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

// ---------------------------------------------------------------------------
// Fixed scratch for awq_scale_search_noalloc.  Some callers cannot allocate device
// memory at the point where they quantise (an allocator-less runtime, a memory
// pool that is already fully carved up, a process that must not grow its
// footprint after start-up), so this entry point keeps its scratch in a
// file-scope device array instead of asking for a workspace.  Every device that
// loads the library holds these bytes until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = (size_t)12 << 20;   // 12 MiB
constexpr int kNoAllocMaxK = 16384;
constexpr int kNoAllocMaxM = 1 << 20;

struct NoAllocScratch {
    bool ready = false;
    void* ptr = nullptr;
};
NoAllocScratch g_noalloc[kMaxDevices];

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
awq_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return AWQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    NoAllocScratch& s = g_noalloc[dev];
    if (!s.ready) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return AWQ_ERR_CUDA;
        s.ptr = p;
        s.ready = true;
    }
    *out = s.ptr;
    return AWQ_OK;
}

}  // namespace

extern "C" {

const char* awq_status_string(awq_status s) {
    switch (s) {
        case AWQ_OK: return "AWQ_OK";
        case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG: invalid argument (null/misaligned pointer or bad size)";
        case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED: configuration not supported";
        case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE: workspace too small";
        case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA: a CUDA call or kernel launch failed";
        case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT: a bounded device wait ran out";
        case AWQ_ERR_RANGE: return "AWQ_ERR_RANGE: a dequantised weight of the fp16 GEMM path is not finite in fp16";
    }
    return "AWQ_ERR_UNKNOWN";
}

int32_t awq_abi_version(void) { return 2; }

awq_status awq_quantize_pack(const uint16_t* W, const uint16_t* s, int32_t N, int32_t K, awq_quant_config cfg,
                             uint32_t* qweight, uint16_t* scales, uint32_t* qzeros, void* stream) {
    awq_status st = check_config(cfg);
    if (st != AWQ_OK) return st;
    st = check_shape(N, K, cfg);
    if (st != AWQ_OK) return st;
    if (!W || !qweight || !scales) return AWQ_ERR_INVALID_ARG;
    if (cfg.zero_point && !qzeros) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(qweight) || (s && !aligned16(s))) return AWQ_ERR_INVALID_ARG;
    const long long blocks = (long long)ceil_div(N, kQuantRows) * ceil_div(K, kQuantChunk);
    if (blocks > 0x7fffffffLL) return AWQ_ERR_UNSUPPORTED;
    quantize_pack_kernel<<<(unsigned)blocks, kQuantThreads, 0, (cudaStream_t)stream>>>(
        W, s, N, K, cfg.q_group_size, cfg.zero_point, qweight, scales, cfg.zero_point ? qzeros : nullptr);
    stream_order_kernel<<<1, 32, 0, (cudaStream_t)stream>>>();
    return launch_status();
}

awq_status awq_fold_inverse_scale(const uint16_t* X, const uint16_t* s, int32_t M, int32_t K, uint16_t* X_out,
                                  void* stream) {
    if (!X || !s || !X_out || M <= 0 || K <= 0 || (K & 7)) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(s) || !aligned16(X_out)) return AWQ_ERR_INVALID_ARG;
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    const long long units = (long long)M * K / 8;
    long long grid = (units + 255) / 256;
    if (grid > 8LL * d.sms) grid = 8LL * d.sms;
    fold_inverse_scale_kernel<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(X, s, M, K, X_out);
    return launch_status();
}

awq_status awq_linear_gemv(const uint16_t* X, int32_t M, const uint32_t* qweight, const uint16_t* scales,
                           const uint32_t* qzeros, int32_t N, int32_t K, awq_quant_config cfg, uint16_t* Y,
                           void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    awq_status st = check_linear(X, M, qweight, scales, qzeros, N, K, cfg, Y);
    if (st != AWQ_OK) return st;
    if (M > 8) return AWQ_ERR_UNSUPPORTED;
    return launch_gemv(X, M, qweight, scales, qzeros, N, K, cfg, Y, (cudaStream_t)stream);
}

awq_status awq_linear_gemm(const uint16_t* X, int32_t M, const uint32_t* qweight, const uint16_t* scales,
                           const uint32_t* qzeros, int32_t N, int32_t K, awq_quant_config cfg, uint16_t* Y,
                           void* ws, size_t ws_bytes, void* stream) {
    (void)ws;
    (void)ws_bytes;
    awq_status st = check_linear(X, M, qweight, scales, qzeros, N, K, cfg, Y);
    if (st != AWQ_OK) return st;
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    return launch_gemm_w4a16(X, M, qweight, scales, qzeros, N, K, cfg.q_group_size, cfg.zero_point, Y,
                             (cudaStream_t)stream, d.sms);
}

size_t awq_workspace_bytes(int32_t op, int32_t M, int32_t N, int32_t K, awq_quant_config cfg) {
    if (op == AWQ_OP_SCALE_SEARCH) return search_workspace_bytes(M, N, K, cfg.q_group_size, 64);
    return 0;
}

awq_status awq_scale_search(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N, int32_t K,
                            awq_quant_config cfg, int32_t n_grid, uint16_t* s_out, double* losses_out,
                            int32_t* best_index_out, void* ws, size_t ws_bytes, void* stream) {
    awq_status st = check_config(cfg);
    if (st != AWQ_OK) return st;
    st = check_shape(N, K, cfg);
    if (st != AWQ_OK) return st;
    if (M <= 0 || n_grid < 1 || n_grid > 64) return AWQ_ERR_INVALID_ARG;
    if (!X || !W || !s_out || !ws) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(W) || !aligned16(s_out) || !aligned16(ws)) return AWQ_ERR_INVALID_ARG;
    if (ws_bytes < search_workspace_bytes(M, N, K, cfg.q_group_size, n_grid)) return AWQ_ERR_WORKSPACE;
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    return run_scale_search(X, M, W, N, K, cfg.q_group_size, cfg.zero_point, n_grid, s_out, losses_out,
                            best_index_out, ws, (cudaStream_t)stream, d.sms);
}

awq_status awq_scale_search_noalloc(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N, int32_t K,
                                    awq_quant_config cfg, int32_t n_grid, uint16_t* s_out, double* losses_out,
                                    int32_t* best_index_out, void* stream) {
    awq_status st = check_config(cfg);
    if (st != AWQ_OK) return st;
    st = check_shape(N, K, cfg);
    if (st != AWQ_OK) return st;
    if (M <= 0 || n_grid < 1 || n_grid > kSearchMaxGrid) return AWQ_ERR_INVALID_ARG;
    if (!X || !W || !s_out) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(W) || !aligned16(s_out)) return AWQ_ERR_INVALID_ARG;
    if (K > kNoAllocMaxK || M > kNoAllocMaxM) return AWQ_ERR_UNSUPPORTED;   // beyond the fixed scratch
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != AWQ_OK) return st;
    const ChunkedSearchLayout L = chunked_search_layout(scratch, kNoAllocScratchBytes, M, N, K);
    if (L.nc <= 0) return AWQ_ERR_UNSUPPORTED;
    return run_scale_search_chunked(X, M, W, N, K, cfg.q_group_size, cfg.zero_point, n_grid, s_out, losses_out,
                                    best_index_out, L, (cudaStream_t)stream);
}

awq_status awq_check_bounded_wait(void* stream) {
    awq::sm100::bounded_wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>();
    return launch_status();
}

awq_status awq_device_error(void* stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return AWQ_ERR_CUDA;
    unsigned word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return AWQ_ERR_CUDA;
    if (word == 0) return AWQ_OK;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return AWQ_ERR_CUDA;
    return (word & kErrTimeout) ? AWQ_ERR_TIMEOUT : AWQ_ERR_RANGE;
}

}  // extern "C"
