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
#include "gemv_launch.cuh"
#include "quantize.cuh"
#include "gemm_sm100.cuh"
#include "search.cuh"
#include "clip.cuh"

using namespace awq;

namespace {

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
    uint32_t* qz = cfg.zero_point ? qzeros : nullptr;
    const cudaStream_t st_ = (cudaStream_t)stream;
    switch (cfg.q_group_size) {
        case 32: quantize_pack_kernel<32><<<(unsigned)blocks, kQuantThreads, 0, st_>>>(W, s, N, K, cfg.zero_point, qweight, scales, qz); break;
        case 64: quantize_pack_kernel<64><<<(unsigned)blocks, kQuantThreads, 0, st_>>>(W, s, N, K, cfg.zero_point, qweight, scales, qz); break;
        case 128: quantize_pack_kernel<128><<<(unsigned)blocks, kQuantThreads, 0, st_>>>(W, s, N, K, cfg.zero_point, qweight, scales, qz); break;
        default: quantize_pack_kernel<256><<<(unsigned)blocks, kQuantThreads, 0, st_>>>(W, s, N, K, cfg.zero_point, qweight, scales, qz); break;
    }
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
    awq_status st = check_linear(X, M, qweight, scales, qzeros, N, K, cfg, Y);
    if (st != AWQ_OK) return st;
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    if (ws && !aligned16(ws)) return AWQ_ERR_INVALID_ARG;
    return launch_gemm_w4a16(X, M, qweight, scales, qzeros, N, K, cfg.q_group_size, cfg.zero_point, Y,
                             (cudaStream_t)stream, d.sms, ws, ws ? ws_bytes : 0);
}

size_t awq_workspace_bytes(int32_t op, int32_t M, int32_t N, int32_t K, awq_quant_config cfg) {
    if (op == AWQ_OP_SCALE_SEARCH) return search_workspace_bytes(M, N, K, cfg.q_group_size, 64);
    if (op == AWQ_OP_GEMM) {
        DeviceInfo d;
        return gemm_workspace_bytes(M, N, K, device_info(d) ? d.sms : 148);
    }
    return 0;
}

}  // extern "C"

namespace {

awq_status scale_search_common(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N, int32_t K,
                               awq_quant_config cfg, bool duo, int32_t n_grid, uint16_t* s_out, double* losses_out,
                               int32_t* best_index_out, void* ws, size_t ws_bytes, void* stream) {
    awq_status st = check_config(cfg);
    if (st != AWQ_OK) return st;
    st = check_shape(N, K, cfg);
    if (st != AWQ_OK) return st;
    if (M <= 0 || n_grid < 1 || n_grid > kSearchMaxGrid) return AWQ_ERR_INVALID_ARG;
    if (!X || !W || !s_out || !ws) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(W) || !aligned16(s_out) || !aligned16(ws)) return AWQ_ERR_INVALID_ARG;
    if (ws_bytes < search_workspace_bytes(M, N, K, cfg.q_group_size, n_grid)) return AWQ_ERR_WORKSPACE;
    return run_scale_search(X, M, W, N, K, cfg.q_group_size, cfg.zero_point, duo, n_grid, s_out, losses_out,
                            best_index_out, ws, (cudaStream_t)stream);
}

}  // namespace

extern "C" {

awq_status awq_scale_search(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N, int32_t K,
                            awq_quant_config cfg, int32_t n_grid, uint16_t* s_out, double* losses_out,
                            int32_t* best_index_out, void* ws, size_t ws_bytes, void* stream) {
    return scale_search_common(X, M, W, N, K, cfg, false, n_grid, s_out, losses_out, best_index_out, ws, ws_bytes,
                               stream);
}

awq_status awq_scale_search_duo(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N, int32_t K,
                                awq_quant_config cfg, int32_t n_grid, uint16_t* s_out, double* losses_out,
                                int32_t* best_index_out, void* ws, size_t ws_bytes, void* stream) {
    return scale_search_common(X, M, W, N, K, cfg, true, n_grid, s_out, losses_out, best_index_out, ws, ws_bytes,
                               stream);
}

size_t awq_apply_clip_workspace_bytes(int32_t M, int32_t N, int32_t K, awq_quant_config cfg, int32_t n_clip) {
    if (check_config(cfg) != AWQ_OK || K % cfg.q_group_size) return 0;
    return clip_workspace_bytes(M, N, K, cfg.q_group_size, n_clip);
}

awq_status awq_apply_clip(const uint16_t* X, int32_t M, const uint16_t* W, const uint16_t* s, int32_t N, int32_t K,
                          awq_quant_config cfg, int32_t n_grid, int32_t n_clip, uint32_t* qweight, uint16_t* scales,
                          uint32_t* qzeros, uint8_t* clip_index_out, double* err_out, void* ws, size_t ws_bytes,
                          void* stream) {
    awq_status st = check_config(cfg);
    if (st != AWQ_OK) return st;
    st = check_shape(N, K, cfg);
    if (st != AWQ_OK) return st;
    if (M <= 0 || n_grid < 1 || n_clip < 1 || n_clip > n_grid || n_clip > kClipMaxRatios) return AWQ_ERR_INVALID_ARG;
    if (!X || !W || !qweight || !scales || !ws) return AWQ_ERR_INVALID_ARG;
    if (cfg.zero_point && !qzeros) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(W) || !aligned16(qweight) || !aligned16(ws) || (s && !aligned16(s)))
        return AWQ_ERR_INVALID_ARG;
    if (ws_bytes < clip_workspace_bytes(M, N, K, cfg.q_group_size, n_clip)) return AWQ_ERR_WORKSPACE;
    DeviceInfo d;
    if (!device_info(d)) return AWQ_ERR_CUDA;
    return run_apply_clip(X, M, W, s, N, K, cfg.q_group_size, cfg.zero_point, n_grid, n_clip, qweight, scales,
                          qzeros, clip_index_out, err_out, ws, (cudaStream_t)stream, d.sms);
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
    const ChunkedSearchLayout L = chunked_search_layout(scratch, kNoAllocScratchBytes, M, N, K, cfg.q_group_size);
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
