// moe_forward_noalloc: the whole MoE block without any device allocation.
//
// Some callers cannot call cudaMalloc at all: frameworks whose custom
// allocator owns every byte of device memory, or plugins loaded into a host
// that forbids allocation from library code.  For them this entry point takes its scratch
// memory from one file-scope __device__ array of fixed size (every GPU that
// loads the library holds it until process exit).  The caller still passes
// every input, the weights and the output.
//
// The scratch array's host-side name is only a stand-in: host code gets the
// device address with cudaGetSymbolAddress, once per device, with that device
// current; kernels receive that pointer.  The first call on a device does this
// set-up, so make the first call outside any stream capture.
//
// Calls share the array: two calls that overlap on the GPU (different
// streams, or different host threads on the same device) race on it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "host_plan.cuh"
#include "kernels.cuh"
#include "moe_b200.h"

namespace moe {
cudaError_t launch_route(const RouteParams &p, cudaStream_t s);
cudaError_t launch_group(const GroupParams &p, cudaStream_t s);
bool route_group_small_fits(const RouteParams &p);
cudaError_t launch_route_group_small(const RouteParams &rp, const GroupParams &gp, unsigned int *bar,
                                     unsigned long long wait_limit_ns, cudaStream_t s);
cudaError_t launch_combine(const uint16_t *x, const float *orows, const int *pair_row, uint16_t *y, int T, int d, int k,
                           cudaStream_t s);
cudaError_t launch_expert_gemm(int mode, const GemmParams &p, int grid, int smem, cudaStream_t s);
}  // namespace moe

using namespace moe;

namespace {

// 8 MiB of scratch: enough for decode-sized batches of the gpt-oss layers
// (up to 64 tokens, top-4, d_model = d_ff = 2880 needs about 7.96 MiB with 128
// experts).
constexpr size_t kScratchBytes = 8u << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
unsigned char *g_scratch_ptr[kMaxDevices];   // device address of g_noalloc_scratch, per device
int g_num_sms[kMaxDevices];

size_t r256(size_t v) { return (v + 255) & ~size_t(255); }

bool a16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool a32(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// Device address of the scratch array on the current device (set up once per device).
int scratch_for_current_device(unsigned char **ptr, int *num_sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
        if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_num_sms[dev] = prop.multiProcessorCount;
        g_scratch_ptr[dev] = static_cast<unsigned char *>(p);
    }
    *ptr = g_scratch_ptr[dev];
    *num_sms = g_num_sms[dev];
    return MOE_OK;
}

// The grouped GEMM launch of one expert stage on scratch-backed buffers.
int launch_gemm_stage(int mode, int T, int k, int d, int F, int E, int num_sms, const uint8_t *codes,
                      const uint8_t *scales, const uint16_t *bias, const CUtensorMap *map_b, const uint32_t *b_sf,
                      const int *counts, const int *offsets, const int *tiles, const int *row_token,
                      const float *row_w, uint8_t *h_q, uint32_t *h_sf, float *out_rows, unsigned int *err,
                      cudaStream_t stream) {
    GemmParams p;
    memset(&p, 0, sizeof p);
    int grid = 0, smem = 0;
    int rc = plan_gemm(p, mode, T, k, d, F, E, T * k, num_sms, &grid, &smem);
    if (rc) return rc;
    if (p.K_main >= 128) {
        const bool ok = mode == MODE_UP ? encode_a_up(&p.map_a, codes, E, F, d, p.K_main)
                                        : encode_a_down(&p.map_a, codes, E, d, F, p.K_main);
        if (!ok) return MOE_ERR_CUDA;
    }
    p.map_b = *map_b;
    p.codes = codes;
    p.scales = scales;
    p.bias = bias;
    p.b_sf = b_sf;
    p.counts = counts;
    p.offsets = offsets;
    p.tiles = tiles;
    p.row_token = row_token;
    p.row_w = row_w;
    p.h_q = h_q;
    p.h_sf = reinterpret_cast<uint8_t *>(h_sf);
    p.out_rows = out_rows;
    p.err = err;
    p.wait_limit_ns = 2000000000ull;
    return launch_expert_gemm(mode, p, grid, smem, stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

MOE_API int moe_forward_noalloc(int T, int d_model, int d_ff, int n_experts, int top_k, float eps,
                                const uint16_t *x, const uint16_t *router_w, const float *router_b,
                                const uint8_t *w13_codes, const uint8_t *w13_scales, const uint16_t *b13,
                                const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                                const uint16_t *norm_scale, uint16_t *y, void *stream) {
    const int d = d_model, F = d_ff, E = n_experts, k = top_k;
    if (T < 0 || T > MOE_NOALLOC_MAX_TOKENS) return MOE_ERR_ARG;
    if (d < 64 || d > 6144 || d % 64 || F < 64 || F > 6144 || F % 64) return MOE_ERR_ARG;
    if (E < 1 || E > 256 || k < 1 || k > 8 || k > E || !(eps >= 0.0f)) return MOE_ERR_ARG;
    if (T == 0) return MOE_OK;
    if (!a16(x) || !a16(router_w) || !a16(router_b) || !a32(w13_codes) || !a16(w13_scales) || !a16(b13) ||
        !a32(w2_codes) || !a16(w2_scales) || !a16(b2) || !a16(norm_scale) || !a16(y) || y == x)
        return MOE_ERR_ARG;

    // carve the scratch; reject shapes that do not fit
    const size_t P = (size_t)T * k;
    const int Kd = round_up_128(d), Kf = round_up_128(F);
    const size_t sizes[] = {(size_t)T * d * 4, P * 4, P * 4, (size_t)E * 4, (size_t)(E + 1) * 4,
                            (size_t)(E + 1) * 4, P * 4, P * 4, P * 4,
                            3 * P * Kd, (size_t)(Kd / 128) * 2 * P * 4, 3 * P * Kf, (size_t)(Kf / 128) * 2 * P * 4,
                            P * d * 4, 64, (size_t)T * E * 4, (size_t)T * 4};
    size_t total = 0;
    for (size_t v : sizes) total += r256(v);
    if (total > kScratchBytes) return MOE_ERR_ARG;

    unsigned char *base = nullptr;
    int num_sms = 0;
    int rc = scratch_for_current_device(&base, &num_sms);
    if (rc) return rc;
    unsigned char *ptrs[sizeof(sizes) / sizeof(sizes[0])];
    for (size_t i = 0; i < sizeof(sizes) / sizeof(sizes[0]); ++i) {
        ptrs[i] = base;
        base += r256(sizes[i]);
    }
    float *xn = reinterpret_cast<float *>(ptrs[0]);
    int *topk_idx = reinterpret_cast<int *>(ptrs[1]);
    float *topk_w = reinterpret_cast<float *>(ptrs[2]);
    int *counts = reinterpret_cast<int *>(ptrs[3]);
    int *offsets = reinterpret_cast<int *>(ptrs[4]);
    int *tiles = reinterpret_cast<int *>(ptrs[5]);
    int *row_token = reinterpret_cast<int *>(ptrs[6]);
    float *row_w = reinterpret_cast<float *>(ptrs[7]);
    int *pair_row = reinterpret_cast<int *>(ptrs[8]);
    uint8_t *xq = reinterpret_cast<uint8_t *>(ptrs[9]);
    uint32_t *xsf = reinterpret_cast<uint32_t *>(ptrs[10]);
    uint8_t *hq = reinterpret_cast<uint8_t *>(ptrs[11]);
    uint32_t *hsf = reinterpret_cast<uint32_t *>(ptrs[12]);
    float *orows = reinterpret_cast<float *>(ptrs[13]);
    unsigned int *err = reinterpret_cast<unsigned int *>(ptrs[14]);
    float *logits = reinterpret_cast<float *>(ptrs[15]);
    unsigned int *tok_done = reinterpret_cast<unsigned int *>(ptrs[16]);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nb = token_block_rows(T);
    const int planes = gemm_b_planes(nb <= 64 ? 1 : 0);
    CUtensorMap map_xq, map_hq;
    if (!encode_bq(&map_xq, xq, (int)P, Kd, nb, planes) || !encode_bq(&map_hq, hq, (int)P, Kf, nb, planes))
        return MOE_ERR_CUDA;
    // the error word with the grid barrier words beside it, and the route kernel's per-token
    // counters, must start at zero on every call (the array keeps whatever the previous call,
    // of any shape, left)
    if (cudaMemsetAsync(err, 0, 64, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(tok_done, 0, (size_t)T * sizeof(unsigned int), s) != cudaSuccess) return MOE_ERR_CUDA;

    RouteParams rp;
    rp.x = x;
    rp.norm_scale = norm_scale;
    rp.router_w = router_w;
    rp.router_b = router_b;
    rp.T = T;
    rp.d = d;
    rp.E = E;
    rp.k = k;
    rp.eps = eps;
    rp.xn = xn;
    rp.topk_idx = topk_idx;
    rp.topk_w = topk_w;
    rp.logits = logits;
    rp.tok_done = tok_done;

    GroupParams gp;
    gp.topk_idx = topk_idx;
    gp.topk_w = topk_w;
    gp.P = (int)P;
    gp.k = k;
    gp.E = E;
    gp.nb_rows = nb;
    gp.counts = counts;
    gp.offsets = offsets;
    gp.tiles = tiles;
    gp.row_token = row_token;
    gp.row_w = row_w;
    gp.pair_row = pair_row;
    gp.err = err;
    gp.xn = xn;
    gp.xq = xq;
    gp.xsf = xsf;
    gp.P_max = (int)P;
    gp.d = d;
    gp.Kd = Kd;
    gp.h_ready = nullptr;
    gp.n_h_ready = 0;
    if (route_group_small_fits(rp)) {
        // route and group in one launch; its grid barrier words sit after the error word
        if (launch_route_group_small(rp, gp, err + 8, 2000000000ull, s) != cudaSuccess) return MOE_ERR_CUDA;
    } else {
        if (launch_route(rp, s) != cudaSuccess) return MOE_ERR_CUDA;
        if (launch_group(gp, s) != cudaSuccess) return MOE_ERR_CUDA;
    }

    rc = launch_gemm_stage(MODE_UP, T, k, d, F, E, num_sms, w13_codes, w13_scales, b13, &map_xq, xsf, counts,
                           offsets, tiles, row_token, row_w, hq, hsf, orows, err, s);
    if (rc) return rc;
    rc = launch_gemm_stage(MODE_DOWN, T, k, d, F, E, num_sms, w2_codes, w2_scales, b2, &map_hq, hsf, counts,
                           offsets, tiles, row_token, row_w, hq, hsf, orows, err, s);
    if (rc) return rc;
    return launch_combine(x, orows, pair_row, y, T, d, k, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
