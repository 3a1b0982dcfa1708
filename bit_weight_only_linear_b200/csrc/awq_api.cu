// C ABI of the AWQ W4A16 library: argument checks, launch configuration, and the
// entry points declared in include/awq.h.  The whole library is one translation
// unit (this file includes the kernel headers), so the device error word and the
// kernels share one module.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

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

template <int WT, bool ONE>
awq_status launch_gemv(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                       const uint32_t* qzeros, int N, int K, const awq_quant_config& cfg, uint16_t* Y,
                       cudaStream_t st) {
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    const int nsteps = K / (32 * WT);
    const size_t smem = GemvSmem::bytes(M, K, nsteps);
    if (smem > (size_t)d.max_smem_optin) return AWQ_ERR_UNSUPPORTED;
    auto kern = gemv_mma_kernel<WT, ONE>;
    int occ = 0;
    if (!kernel_occupancy((const void*)kern, kGemvThreads, smem, occ) || occ < 1) return AWQ_ERR_CUDA;
    // persistent grid: at most one wave, row-group iterations spread evenly over the CTAs
    constexpr int UK = kGemvUnitWords / WT;
    const int units = ceil_div(nsteps, UK);
    const int slots = d.sms * occ;
    const int ks = gemv_ks(units, ceil_div(N, kGemvRows), slots);
    const int rpi = kGemvWarps / ks;
    const int n_it = ceil_div(ceil_div(N, kGemvRows), rpi);
    const int per_cta = ceil_div(n_it, slots);
    const int grid = ceil_div(n_it, per_cta);
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(grid);
    lc.blockDim = dim3(kGemvThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    if (cudaLaunchKernelEx(&lc, kern, X, M, qweight, scales, qzeros, N, K, (int)cfg.q_group_size,
                           (int)cfg.zero_point, ks, Y) != cudaSuccess)
        return AWQ_ERR_CUDA;
    return launch_status();
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

template <int G, bool ONE>
awq_status launch_gemv_tma(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                           const uint32_t* qzeros, int N, int K, const awq_quant_config& cfg, uint16_t* Y,
                           cudaStream_t st) {
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    int S = 0, PR = 0, ctas = 0;
    if (!pick_gemv_tma(d, M, N, K, G, S, PR, ctas)) return AWQ_ERR_UNSUPPORTED;
    const size_t smem = GemvTmaSmem(M, K, G, S, PR).bytes();
    // qweight [N][K/8] words viewed as {16 words, N rows, K/128 blocks}
    CUtensorMap tq;
    if (!make_tmap_3d(&tq, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT32, 16, (uint64_t)N, (uint64_t)(K / 128),
                      (uint64_t)K / 2, 64, 16, kGemvRows, kTmaKC / 128))
        return AWQ_ERR_CUDA;
    auto kern = gemv_tma_kernel<G, ONE>;
    int occ = 0;
    if (!kernel_occupancy((const void*)kern, kTmaThreads, smem, occ) || occ < 1) return AWQ_ERR_CUDA;
    // one CTA per resident slot, row groups dealt round-robin
    const int n_rg = N / kGemvRows;
    const int slots = d.sms * occ;
    const int grid = n_rg < slots ? n_rg : slots;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(grid);
    lc.blockDim = dim3(kTmaThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    if (cudaLaunchKernelEx(&lc, kern, tq, X, M, scales, qzeros, N, K, (int)cfg.zero_point, Y, S, PR) !=
        cudaSuccess)
        return AWQ_ERR_CUDA;
    return launch_status();
}

template <bool ONE>
awq_status dispatch_gemv(const uint16_t* X, int M, const uint32_t* qweight, const uint16_t* scales,
                         const uint32_t* qzeros, int N, int K, const awq_quant_config& cfg, uint16_t* Y,
                         cudaStream_t s) {
    // every row group full, K in whole 128-code blocks, parameters 16-byte aligned and
    // the staging fits: TMA path
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    if (N % kGemvRows == 0 && K % 128 == 0 && (uintptr_t)scales % 16 == 0 &&
        (!cfg.zero_point || (uintptr_t)qzeros % 16 == 0)) {
        int S = 0, PR = 0, ctas = 0;
        if (aligned16(X) && pick_gemv_tma(d, M, N, K, cfg.q_group_size, S, PR, ctas)) {
#define AWQ_GEMV_TMA(GG) return launch_gemv_tma<GG, ONE>(X, M, qweight, scales, qzeros, N, K, cfg, Y, s)
            switch (cfg.q_group_size) {
                case 32: AWQ_GEMV_TMA(32);
                case 64: AWQ_GEMV_TMA(64);
                case 128: AWQ_GEMV_TMA(128);
                default: AWQ_GEMV_TMA(256);
            }
#undef AWQ_GEMV_TMA
        }
    }
    switch (cfg.q_group_size) {
        case 32: return launch_gemv<1, ONE>(X, M, qweight, scales, qzeros, N, K, cfg, Y, s);
        case 64: return launch_gemv<2, ONE>(X, M, qweight, scales, qzeros, N, K, cfg, Y, s);
        default: return launch_gemv<4, ONE>(X, M, qweight, scales, qzeros, N, K, cfg, Y, s);
    }
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
    }
    return "AWQ_ERR_UNKNOWN";
}

int32_t awq_abi_version(void) { return 1; }

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
    cudaStream_t s = (cudaStream_t)stream;
    return M == 1 ? dispatch_gemv<true>(X, M, qweight, scales, qzeros, N, K, cfg, Y, s)
                  : dispatch_gemv<false>(X, M, qweight, scales, qzeros, N, K, cfg, Y, s);
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
    return AWQ_ERR_TIMEOUT;
}

}  // extern "C"
