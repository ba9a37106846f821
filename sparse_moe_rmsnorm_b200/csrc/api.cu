// C ABI of the B200 MoE block: context and workspace management, argument
// validation, TMA descriptor encoding and the stage launches (moe_forward's
// decode-sized path fuses route + group and the two GEMMs into one launch each).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "moe_b200.h"
#include "host_plan.cuh"
#include "kernels.cuh"

namespace moe {
cudaError_t launch_route(const RouteParams &p, cudaStream_t s);
cudaError_t launch_group(const GroupParams &p, cudaStream_t s);
bool route_group_small_fits(const RouteParams &p);
cudaError_t launch_route_group_small(const RouteParams &rp, const GroupParams &gp, unsigned int *bar,
                                     unsigned long long wait_limit_ns, cudaStream_t s);
cudaError_t launch_combine(const uint16_t *x, const float *orows, const int *pair_row, uint16_t *y, int T, int d, int k,
                           cudaStream_t s);
cudaError_t launch_decode(const uint8_t *codes, const uint8_t *scales, int R, int K, float *out, cudaStream_t s);
cudaError_t launch_selftest_wait(unsigned int *err, unsigned long long limit_ns, cudaStream_t s);
cudaError_t launch_expert_gemm(int mode, const GemmParams &p, int grid, int smem, cudaStream_t s);
cudaError_t launch_expert_ffn(const GemmParams &pu, const GemmParams &pd, int grid, int smem, cudaStream_t s);
cudaError_t launch_pass_plan(const uint8_t *w13_scales, const uint8_t *w2_scales, int E, int d, int F,
                             uint8_t *up_pass, uint8_t *down_pass, cudaStream_t s);
}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// the unpacked-type TMA of the weight codes needs a 32-byte aligned base
bool aligned32(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace

struct moe_ctx {
    moe_shape_t shape;
    int device;
    int num_sms;
    void *ws;
    size_t ws_bytes;
    int Kd, Kf;             // d_model and d_ff rounded up to 128
    float *xn;              // fp32 [T_max, d] normalised tokens
    int *topk_idx;
    float *topk_w;
    float *logits;          // fp32 [T_max, E] router logits (decode-sized route path)
    unsigned int *tok_done; // [T_max] per-token CTA counter of that path (zero between calls)
    int *counts, *offsets, *tiles;
    int *row_token;
    float *row_w;
    int *pair_row;
    uint8_t *xq;            // gate/up B: three E4M3 planes [3][P_max][Kd] of the expert-sorted tokens
    uint32_t *xsf;          // their E8M0 scales [Kd/128][2][P_max] (hi/lo2, lo)
    uint8_t *hq;            // down B: three E4M3 planes [3][P_max][Kf] of h
    uint32_t *hsf;          // [Kf/128][2][P_max]
    float *orows;           // weighted expert output per expert-sorted row
    uint8_t *up_pass;       // [E][F/64] passes over K of each gate/up weight block (large batches)
    uint8_t *down_pass;     // [E][DOWN_PASS_STRIDE] ... of each down weight block
    unsigned int *h_ready;  // [E + P_max/16 + 1] the fused decode GEMM's per-token-block counters
    unsigned int *err;
    unsigned long long wait_limit_ns;
    // B tensor maps, one per token-block height (16 * (i + 1) rows), made on first use
    CUtensorMap map_xq[GEMM_NB_MAX / 16];
    CUtensorMap map_hq[GEMM_NB_MAX / 16];
    bool have_xq[GEMM_NB_MAX / 16], have_hq[GEMM_NB_MAX / 16];
    const void *w13_ptr;
    CUtensorMap map_w13;
    const void *w2_ptr;
    CUtensorMap map_w2;
};

namespace {

struct Buf {
    void *ptr;
    size_t bytes;
};

Buf ws_buffer(moe_ctx *c, int which) {
    const moe_shape_t &s = c->shape;
    const size_t T = (size_t)s.T_max, P = T * s.top_k, E = s.n_experts;
    switch (which) {
        case MOE_WS_XN: return {c->xn, T * s.d_model * 4};
        case MOE_WS_TOPK_IDX: return {c->topk_idx, P * 4};
        case MOE_WS_TOPK_W: return {c->topk_w, P * 4};
        case MOE_WS_COUNTS: return {c->counts, E * 4};
        case MOE_WS_OFFSETS: return {c->offsets, (E + 1) * 4};
        case MOE_WS_ROW_TOKEN: return {c->row_token, P * 4};
        case MOE_WS_ROW_W: return {c->row_w, P * 4};
        case MOE_WS_H: return {c->hq, 3 * P * c->Kf};
        case MOE_WS_OUT_ROWS: return {c->orows, P * s.d_model * 4};
        case MOE_WS_TILES: return {c->tiles, (E + 1) * 4};
        case MOE_WS_PAIR_ROW: return {c->pair_row, P * 4};
        case MOE_WS_XPERM: return {c->xq, 3 * P * c->Kd};
        case MOE_WS_XSF: return {c->xsf, (size_t)(c->Kd / 128) * 2 * P * 4};
        case MOE_WS_HSF: return {c->hsf, (size_t)(c->Kf / 128) * 2 * P * 4};
        default: return {nullptr, 0};
    }
}

int check_call(moe_ctx *c, int T, int top_k) {
    if (!c) return MOE_ERR_ARG;
    if (T < 0 || T > c->shape.T_max) return MOE_ERR_ARG;
    if (top_k < 1 || top_k > c->shape.top_k) return MOE_ERR_ARG;
    return MOE_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// The parameters, grid and shared memory of one grouped GEMM launch (and, for the
// gate/up GEMM of large batches, the launch of the pass plan both GEMMs read).
int gemm_prepare(moe_ctx *c, int mode, int T, int top_k, const uint8_t *codes, const uint8_t *scales,
                 const uint16_t *bias, const uint8_t *w2_scales, cudaStream_t stream, GemmParams &p, int &grid_out,
                 int &smem_out) {
    const moe_shape_t &s = c->shape;
    memset(&p, 0, sizeof p);
    const int E = s.n_experts, d = s.d_model, F = s.d_ff;
    const int P_max = s.T_max * s.top_k;
    int grid = 0, smem = 0;
    int rc = plan_gemm(p, mode, T, top_k, d, F, E, P_max, c->num_sms, &grid, &smem);
    if (rc) return rc;
    // the cached B maps of this token-block height
    if (p.nb_rows < 16 || p.nb_rows > GEMM_NB_MAX || p.nb_rows % 16) return MOE_ERR_ARG;
    const int bi = p.nb_rows / 16 - 1;
    if (mode == MODE_UP) {
        if (codes != c->w13_ptr) {
            if (p.K_main >= 128 && !encode_a_up(&c->map_w13, codes, E, F, d, p.K_main)) return MOE_ERR_CUDA;
            c->w13_ptr = codes;
        }
        if (!c->have_xq[bi]) {
            if (!encode_bq(&c->map_xq[bi], c->xq, P_max, c->Kd, p.nb_rows, gemm_b_planes(p.stacked)))
                return MOE_ERR_CUDA;
            c->have_xq[bi] = true;
        }
        p.map_a = c->map_w13;
        p.map_b = c->map_xq[bi];
        p.b_sf = c->xsf;
        p.h_q = c->hq;
        p.h_sf = reinterpret_cast<uint8_t *>(c->hsf);
        // large blocks: the pass table of both GEMMs, from the weights' scale bytes
        if (!p.stacked) {
            if (launch_pass_plan(scales, w2_scales, E, d, F, c->up_pass, c->down_pass, stream) != cudaSuccess)
                return MOE_ERR_CUDA;
            p.item_pass = c->up_pass;
            p.item_pass_stride = F / 64;
            p.down_pass = c->down_pass;
            p.MB_down = (d + GEMM_BM - 1) / GEMM_BM;
        }
    } else {
        if (codes != c->w2_ptr) {
            if (p.K_main >= 128 && !encode_a_down(&c->map_w2, codes, E, d, F, p.K_main)) return MOE_ERR_CUDA;
            c->w2_ptr = codes;
        }
        if (!c->have_hq[bi]) {
            if (!encode_bq(&c->map_hq[bi], c->hq, P_max, c->Kf, p.nb_rows, gemm_b_planes(p.stacked)))
                return MOE_ERR_CUDA;
            c->have_hq[bi] = true;
        }
        p.map_a = c->map_w2;
        p.map_b = c->map_hq[bi];
        p.b_sf = c->hsf;
        p.out_rows = c->orows;
        if (!p.stacked) {                                // written by moe_expert_up's pass plan
            p.item_pass = c->down_pass;
            p.item_pass_stride = DOWN_PASS_STRIDE;
        }
    }
    p.codes = codes;
    p.scales = scales;
    p.bias = bias;
    p.counts = c->counts;
    p.offsets = c->offsets;
    p.tiles = c->tiles;
    p.row_token = c->row_token;
    p.row_w = c->row_w;
    p.err = c->err;
    p.wait_limit_ns = c->wait_limit_ns;
    grid_out = grid;
    smem_out = smem;
    return MOE_OK;
}

int gemm_launch(moe_ctx *c, int mode, int T, int top_k, const uint8_t *codes, const uint8_t *scales,
                const uint16_t *bias, const uint8_t *w2_scales, cudaStream_t stream) {
    GemmParams p;
    int grid = 0, smem = 0;
    const int rc = gemm_prepare(c, mode, T, top_k, codes, scales, bias, w2_scales, stream, p, grid, smem);
    if (rc) return rc;
    return cuda_status(launch_expert_gemm(mode, p, grid, smem, stream));
}

// Both GEMMs of a decode-sized batch in one launch, when both use per-item scale factors and
// d_model == d_ff; MOE_ERR_UNSUPPORTED when they do not (the caller launches them apart).
int ffn_launch(moe_ctx *c, int T, int top_k, const uint8_t *w13_codes, const uint8_t *w13_scales,
               const uint16_t *b13, const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
               cudaStream_t stream) {
    if (c->shape.d_model != c->shape.d_ff) return MOE_ERR_UNSUPPORTED;
    GemmParams pu, pd;
    int grid_u = 0, smem_u = 0, grid_d = 0, smem_d = 0;
    int rc = gemm_prepare(c, MODE_UP, T, top_k, w13_codes, w13_scales, b13, w2_scales, stream, pu, grid_u, smem_u);
    if (rc) return rc;
    rc = gemm_prepare(c, MODE_DOWN, T, top_k, w2_codes, w2_scales, b2, nullptr, stream, pd, grid_d, smem_d);
    if (rc) return rc;
    if (!pu.sf_item || !pd.sf_item || pu.n_stages != pd.n_stages || smem_u != smem_d) return MOE_ERR_UNSUPPORTED;
    pu.h_ready = pd.h_ready = c->h_ready;
    pu.h_target = pd.h_target = 8u * (unsigned)pu.MB;     // every epilogue warp of every gate/up weight block
    const int grid = grid_u + grid_d < c->num_sms ? grid_u + grid_d : c->num_sms;
    return cuda_status(launch_expert_ffn(pu, pd, grid, smem_u, stream));
}


RouteParams route_params(moe_ctx *c, int T, const uint16_t *x, const uint16_t *norm_scale, const uint16_t *router_w,
                         const float *router_b, int top_k) {
    RouteParams p;
    p.x = x;
    p.norm_scale = norm_scale;
    p.router_w = router_w;
    p.router_b = router_b;
    p.T = T;
    p.d = c->shape.d_model;
    p.E = c->shape.n_experts;
    p.k = top_k;
    p.eps = c->shape.eps;
    p.xn = c->xn;
    p.topk_idx = c->topk_idx;
    p.topk_w = c->topk_w;
    p.logits = c->logits;
    p.tok_done = c->tok_done;
    return p;
}

GroupParams group_params(moe_ctx *c, int T, int top_k) {
    GroupParams p;
    p.topk_idx = c->topk_idx;
    p.topk_w = c->topk_w;
    p.P = T * top_k;
    p.k = top_k;
    p.E = c->shape.n_experts;
    p.nb_rows = token_block_rows(T);
    p.counts = c->counts;
    p.offsets = c->offsets;
    p.tiles = c->tiles;
    p.row_token = c->row_token;
    p.row_w = c->row_w;
    p.pair_row = c->pair_row;
    p.err = c->err;
    p.xn = c->xn;
    p.xq = c->xq;
    p.xsf = c->xsf;
    p.P_max = c->shape.T_max * c->shape.top_k;
    p.d = c->shape.d_model;
    p.Kd = c->Kd;
    p.h_ready = c->h_ready;
    p.n_h_ready = c->shape.n_experts + p.P_max / 16 + 1;
    return p;
}

// the grid barrier words of the decode-sized route + group launch: [count, generation], in the
// error word's slot (zero at creation; moe_sync_status clears the slot after an error)
unsigned int *route_group_barrier(moe_ctx *c) { return c->err + 8; }

}  // namespace

extern "C" {

const char *moe_strerror(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_UNSUPPORTED: return "unsupported device (needs compute capability 10.0)";
        case MOE_ERR_NOMEM: return "out of device memory";
        default: return "unknown error";
    }
}

const char *moe_version(void) { return "moe_b200 0.1 (sm_100a)"; }

int moe_init(const moe_shape_t *shape, moe_ctx_t **out) {
    if (!shape || !out) return MOE_ERR_ARG;
    *out = nullptr;
    const moe_shape_t s = *shape;
    if (s.T_max < 1 || s.T_max > (1 << 20)) return MOE_ERR_ARG;
    if (s.d_model < 64 || s.d_model > 6144 || s.d_model % 64) return MOE_ERR_ARG;
    if (s.d_ff < 64 || s.d_ff > 6144 || s.d_ff % 64) return MOE_ERR_ARG;
    if (s.n_experts < 1 || s.n_experts > 256) return MOE_ERR_ARG;
    if (s.top_k < 1 || s.top_k > 8 || s.top_k > s.n_experts) return MOE_ERR_ARG;
    if (!(s.eps >= 0.0f)) return MOE_ERR_ARG;
    if ((long long)s.T_max * s.top_k > (1LL << 30) / 1) return MOE_ERR_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED;
    if (!encode_fn()) return MOE_ERR_CUDA;

    moe_ctx *c = new (std::nothrow) moe_ctx;
    if (!c) return MOE_ERR_NOMEM;
    memset(c, 0, sizeof *c);
    c->shape = s;
    c->device = dev;
    c->num_sms = prop.multiProcessorCount;
    c->wait_limit_ns = 2000000000ull;

    c->Kd = round_up_128(s.d_model);
    c->Kf = round_up_128(s.d_ff);
    const size_t T = (size_t)s.T_max, P = T * s.top_k, E = s.n_experts;
    const size_t sizes[] = {T * s.d_model * 4, P * 4, P * 4, E * 4, (E + 1) * 4, (E + 1) * 4,
                            P * 4, P * 4, P * 4,
                            3 * P * c->Kd, (size_t)(c->Kd / 128) * 2 * P * 4,
                            3 * P * c->Kf, (size_t)(c->Kf / 128) * 2 * P * 4,
                            P * s.d_model * 4, 64, T * E * 4, T * 4, E * (size_t)(s.d_ff / 64),
                            E * (size_t)DOWN_PASS_STRIDE, (E + P / 16 + 1) * 4};
    void **slots[] = {(void **)&c->xn, (void **)&c->topk_idx, (void **)&c->topk_w,
                      (void **)&c->counts, (void **)&c->offsets, (void **)&c->tiles, (void **)&c->row_token,
                      (void **)&c->row_w, (void **)&c->pair_row, (void **)&c->xq, (void **)&c->xsf,
                      (void **)&c->hq, (void **)&c->hsf, (void **)&c->orows, (void **)&c->err,
                      (void **)&c->logits, (void **)&c->tok_done, (void **)&c->up_pass, (void **)&c->down_pass,
                      (void **)&c->h_ready};
    size_t total = 0;
    for (size_t v : sizes) total += round256(v);
    if (cudaMalloc(&c->ws, total) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return MOE_ERR_NOMEM;
    }
    c->ws_bytes = total;
    char *b = static_cast<char *>(c->ws);
    for (size_t i = 0; i < sizeof(sizes) / sizeof(sizes[0]); ++i) {
        *slots[i] = sizes[i] ? b : nullptr;
        b += round256(sizes[i]);
    }
    if (cudaMemset(c->ws, 0, total) != cudaSuccess) {
        cudaFree(c->ws);
        delete c;
        return MOE_ERR_CUDA;
    }
    *out = c;
    return MOE_OK;
}

int moe_destroy(moe_ctx_t *ctx) {
    if (!ctx) return MOE_OK;
    cudaDeviceSynchronize();
    cudaFree(ctx->ws);
    delete ctx;
    return MOE_OK;
}

int moe_route(moe_ctx_t *c, int T, const uint16_t *x, const uint16_t *norm_scale, const uint16_t *router_w,
              const float *router_b, int top_k, void *stream) {
    int rc = check_call(c, T, top_k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned16(x) || !aligned16(norm_scale) || !aligned16(router_w) || !aligned16(router_b)) return MOE_ERR_ARG;
    return cuda_status(launch_route(route_params(c, T, x, norm_scale, router_w, router_b, top_k),
                                    static_cast<cudaStream_t>(stream)));
}

int moe_group(moe_ctx_t *c, int T, int top_k, void *stream) {
    int rc = check_call(c, T, top_k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    return cuda_status(launch_group(group_params(c, T, top_k), static_cast<cudaStream_t>(stream)));
}

int moe_expert_up(moe_ctx_t *c, int T, int top_k, const uint8_t *w13_codes, const uint8_t *w13_scales,
                  const uint16_t *b13, const uint8_t *w2_scales, void *stream) {
    int rc = check_call(c, T, top_k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned32(w13_codes) || !aligned16(w13_scales) || !aligned16(b13) || !aligned16(w2_scales))
        return MOE_ERR_ARG;
    return gemm_launch(c, MODE_UP, T, top_k, w13_codes, w13_scales, b13, w2_scales,
                       static_cast<cudaStream_t>(stream));
}

int moe_expert_down(moe_ctx_t *c, int T, int top_k, const uint8_t *w2_codes, const uint8_t *w2_scales,
                    const uint16_t *b2, void *stream) {
    int rc = check_call(c, T, top_k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned32(w2_codes) || !aligned16(w2_scales) || !aligned16(b2)) return MOE_ERR_ARG;
    return gemm_launch(c, MODE_DOWN, T, top_k, w2_codes, w2_scales, b2, nullptr, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn(moe_ctx_t *c, int T, int top_k, const uint8_t *w13_codes, const uint8_t *w13_scales,
                   const uint16_t *b13, const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                   void *stream) {
    int rc = check_call(c, T, top_k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned32(w13_codes) || !aligned16(w13_scales) || !aligned16(b13) || !aligned32(w2_codes) ||
        !aligned16(w2_scales) || !aligned16(b2))
        return MOE_ERR_ARG;
    if (T > 64 || T * top_k > 512) return MOE_ERR_UNSUPPORTED;
    return ffn_launch(c, T, top_k, w13_codes, w13_scales, b13, w2_codes, w2_scales, b2,
                      static_cast<cudaStream_t>(stream));
}

int moe_finalize(moe_ctx_t *c, int T, int top_k, const uint16_t *x, uint16_t *y, int32_t *topk_idx_out,
                 float *topk_w_out, void *stream) {
    int rc = check_call(c, T, top_k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned16(x) || !aligned16(y) || x == y) return MOE_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rc = cuda_status(launch_combine(x, c->orows, c->pair_row, y, T, c->shape.d_model, top_k, s));
    if (rc) return rc;
    const size_t pk = (size_t)T * top_k;
    if (topk_idx_out && cudaMemcpyAsync(topk_idx_out, c->topk_idx, pk * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (topk_w_out && cudaMemcpyAsync(topk_w_out, c->topk_w, pk * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_forward(moe_ctx_t *c, int T, const uint16_t *x, const uint16_t *router_w, const float *router_b,
                const uint8_t *w13_codes, const uint8_t *w13_scales, const uint16_t *b13,
                const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                const uint16_t *norm_scale, int top_k, uint16_t *y, int32_t *topk_idx_out, float *topk_w_out,
                void *stream) {
    int rc = check_call(c, T, top_k);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(router_b) || !aligned32(w13_codes) ||
        !aligned16(w13_scales) || !aligned16(b13) || !aligned32(w2_codes) || !aligned16(w2_scales) ||
        !aligned16(b2) || !aligned16(norm_scale) || !aligned16(y))
        return MOE_ERR_ARG;
    if (y == x) return MOE_ERR_ARG;
    const RouteParams rp = route_params(c, T, x, norm_scale, router_w, router_b, top_k);
    if (route_group_small_fits(rp)) {
        // decode-sized batches: route and group in one launch, then both GEMMs in one launch (the
        // same outputs as the stages; the route + group launch zeroes the GEMM launch's counters)
        if (launch_route_group_small(rp, group_params(c, T, top_k), route_group_barrier(c), c->wait_limit_ns,
                                     static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return MOE_ERR_CUDA;
        rc = moe_expert_ffn(c, T, top_k, w13_codes, w13_scales, b13, w2_codes, w2_scales, b2, stream);
        if (rc == MOE_OK) return moe_finalize(c, T, top_k, x, y, topk_idx_out, topk_w_out, stream);
        if (rc != MOE_ERR_UNSUPPORTED) return rc;
    } else {
        if ((rc = moe_route(c, T, x, norm_scale, router_w, router_b, top_k, stream))) return rc;
        if ((rc = moe_group(c, T, top_k, stream))) return rc;
    }
    if ((rc = moe_expert_up(c, T, top_k, w13_codes, w13_scales, b13, w2_scales, stream))) return rc;
    if ((rc = moe_expert_down(c, T, top_k, w2_codes, w2_scales, b2, stream))) return rc;
    return moe_finalize(c, T, top_k, x, y, topk_idx_out, topk_w_out, stream);
}

int moe_copy_workspace(moe_ctx_t *c, int which, void *dst, size_t bytes, void *stream) {
    if (!c || !dst) return MOE_ERR_ARG;
    const Buf b = ws_buffer(c, which);
    if (!b.ptr || bytes > b.bytes) return MOE_ERR_ARG;
    if (bytes == 0) return MOE_OK;
    return cuda_status(cudaMemcpyAsync(dst, b.ptr, bytes, cudaMemcpyDefault, static_cast<cudaStream_t>(stream)));
}

int moe_sync_status(moe_ctx_t *c, void *stream) {
    if (!c) return MOE_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int err = 0;
    if (cudaMemcpyAsync(&err, c->err, sizeof err, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    if (err) {
        // the error word and the grid barrier words beside it (a barrier that ran out is left mid-count)
        if (cudaMemsetAsync(c->err, 0, 64, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_ERR_TIMEOUT;
    }
    return MOE_OK;
}

int moe_set_wait_limit_ns(moe_ctx_t *c, unsigned long long ns) {
    if (!c || ns == 0) return MOE_ERR_ARG;
    c->wait_limit_ns = ns;
    return MOE_OK;
}

int moe_selftest_wait_timeout(moe_ctx_t *c, void *stream) {
    if (!c) return MOE_ERR_ARG;
    return cuda_status(launch_selftest_wait(c->err, c->wait_limit_ns, static_cast<cudaStream_t>(stream)));
}

int moe_debug_decode(const uint8_t *codes, const uint8_t *scales, int R, int K, float *out, void *stream) {
    if (!codes || !scales || !out || R < 0 || K < 32 || K % 32) return MOE_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(codes) & 3u) || (K / 2) % 4) return MOE_ERR_ARG;
    return cuda_status(launch_decode(codes, scales, R, K, out, static_cast<cudaStream_t>(stream)));
}

int moe_debug_plan(int mode, int T, int top_k, int d, int F, int E, int P_max, int num_sms, int *out) {
    if (!out || (mode != MODE_UP && mode != MODE_DOWN) || T < 1 || num_sms < 1) return MOE_ERR_ARG;
    if (d < 64 || d > 6144 || d % 64 || F < 64 || F > 6144 || F % 64) return MOE_ERR_ARG;
    if (E < 1 || E > 256 || top_k < 1 || top_k > 8 || top_k > E) return MOE_ERR_ARG;
    if ((long long)T * top_k > P_max || P_max > (1 << 30)) return MOE_ERR_ARG;
    GemmParams p;
    memset(&p, 0, sizeof p);
    int grid = 0, smem = 0;
    const int rc = plan_gemm(p, mode, T, top_k, d, F, E, P_max, num_sms, &grid, &smem);
    if (rc) return rc;
    const int n_st = (p.K + GEMM_KS - 1) / GEMM_KS;
    out[0] = p.nb_rows;
    out[1] = p.stacked;
    out[2] = p.n_stages;
    out[3] = p.sf_item;
    out[4] = grid;
    out[5] = smem;
    out[6] = p.sf_item ? gemm_tmem_cols_item(p.nb_rows, p.stacked, n_st) : gemm_tmem_cols(p.nb_rows, p.stacked, p.n_stages);
    out[7] = p.K_main / GEMM_KS;
    out[8] = n_st;
    out[9] = p.MB;
    return MOE_OK;
}

}  // extern "C"
