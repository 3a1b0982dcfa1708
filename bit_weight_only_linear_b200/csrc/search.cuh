// Activation-aware scale search (placeholder for the kernels; workspace layout is final).
#pragma once

#include "common.cuh"

namespace awq {

constexpr int kSearchMaxGrid = 64;     // n_grid upper bound (s table and losses)
constexpr int kSearchBatch = 8;        // alphas evaluated per pass
constexpr int kSearchTileM = 128;      // calibration tokens per tile
constexpr int kSearchTileN = 128;      // output channels per tile (upper bound on tile count)

struct SearchWorkspace {
    double* colsum;      // [K]
    uint16_t* s_all;     // [kSearchMaxGrid][K]
    uint16_t* dw;        // [kSearchBatch][N][2K]: (Q(Ws)/s - W) * 2^e_n as hi/lo fp16 per 64-channel block
    int32_t* row_exp;    // [kSearchBatch][N]
    double* partial;     // [kSearchBatch][tiles]
    double* losses;      // [kSearchMaxGrid]
    size_t bytes;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

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
    w.dw = reinterpret_cast<uint16_t*>(take((size_t)kSearchBatch * N * 2 * K * 2));
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

inline awq_status run_scale_search(const uint16_t*, int, const uint16_t*, int, int, int, int, int, uint16_t*,
                                   double*, int32_t*, void*, cudaStream_t, int) {
    return AWQ_ERR_UNSUPPORTED;
}

}  // namespace awq
