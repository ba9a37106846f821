// Kernel parameter blocks and launch-side constants shared by api.cu and the
// kernel sources.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

namespace moe {

// Error bits of the device error word.
enum : unsigned int {
    ERR_WAIT_UP = 1u,      // a bounded wait ran out in the gate/up GEMM
    ERR_WAIT_DOWN = 2u,    // ... in the down GEMM
    ERR_WAIT_SELFTEST = 4u,
    ERR_ROUTING = 8u       // an expert index out of range reached the grouping
};

struct RouteParams {
    const uint16_t *x;          // bf16 [T, d]
    const uint16_t *norm_scale; // bf16 [d]
    const uint16_t *router_w;   // bf16 [E, d]
    const float *router_b;      // fp32 [E]
    int T, d, E, k;
    float eps;
    __half *xn16;               // fp16 [T, d] = xn / rho
    float *rho;                 // fp32 [T]
    int *topk_idx;              // [T, k]
    float *topk_w;              // [T, k]
};

struct GroupParams {
    const int *topk_idx;        // [P] = [T, k]
    const float *topk_w;        // [P]
    int P, k, E, nb_rows;
    int *counts;                // [E]
    int *offsets;               // [E+1]
    int *tiles;                 // [E+1] prefix of ceil(counts / nb_rows)
    int *row_token;             // [P]
    float *row_w;               // [P]
    int *pair_row;              // [P] expert-sorted row of pair (token, slot)
    unsigned int *err;
};

// Grouped MXFP4 x fp16 GEMM over (expert, 128-row weight block, token block)
// work items.  MODE_UP: rows are the gate/linear pairs of W13, epilogue is the
// clamped SwiGLU into h.  MODE_DOWN: rows are W2's, epilogue writes the
// routing-weighted expert output rows.
enum { MODE_UP = 0, MODE_DOWN = 1 };

struct GemmParams {
    CUtensorMap map_codes;      // u8 [E][R][K/2], box {128 bytes, 64 (UP) or 128 (DOWN) rows, 1}, 128B swizzle
    CUtensorMap map_b;          // fp16 expert-sorted B, K-blocked [K/64][P_max][64]; 3-D box {64, b_box_rows, b_unit}
    const uint8_t *scales;      // u8 [E][R][K/32]
    const uint16_t *bias;       // bf16 [E][R]
    int K;                      // reduction length
    int R;                      // rows per expert: 2F (UP) or d (DOWN)
    int F;                      // d_ff (UP: gate rows [0,F), linear rows [F,2F))
    int E;
    int MB;                     // weight blocks per expert: F/64 (UP) or ceil(d/128) (DOWN)
    int nb_rows;                // token rows per work item (multiple of 16, <= 256)
    int b_box_rows;             // rows per B TMA box (16..64)
    int b_unit;                 // sub-stages (64-K blocks) per B ring slot: 4 when one box holds the token block, else 1
    int n_b_stages;             // B ring depth (slots)
    int b_stage_bytes;          // bytes of one sub-stage block in a slot: round_up(nb_rows, b_box_rows) * 128
    int b_rows_total;           // P_max: rows of the K-blocked B and h buffers
    int n_c_stages;             // code ring depth (shared-memory stages of 128 rows x 128 bytes)
    int n_a_slots;              // TMEM A slots (32 columns each); accumulators follow them
    int n_iss;                  // MMA-issuing warps, each with its own accumulator
    int n_dec_groups;           // decoder warp groups, 1..3 (with 3, warps 16-19 decode and one epilogue group remains)
    int n_d_bufs;               // accumulator buffer sets (1 or 2)
    const int *counts, *offsets, *tiles;
    const int *row_token;       // [P]
    const float *row_w;         // [P]
    const float *rho;           // [T] (UP)
    void *out;                  // UP: fp16 h [P][F]; DOWN: fp32 weighted outputs [P][d]
    int out_ld;                 // F (UP) or d (DOWN)
    unsigned int *err;
    unsigned long long wait_limit_ns;
};

constexpr int GEMM_THREADS = 672;     // 21 warps
constexpr int GEMM_BM = 128;          // weight rows per work item (TMEM lanes)
constexpr int GEMM_KS = 256;          // K elements per code stage: 128 bytes per row
constexpr int GEMM_KA = 64;           // K elements per TMEM A slot: 32 columns
constexpr int GEMM_SC_MAX = 10;       // code stages, at most
constexpr int GEMM_NA_MAX = 14;       // TMEM A slots, at most
constexpr int GEMM_NB_MAX = 256;      // token rows per work item, at most
constexpr int GEMM_ISS_MAX = 3;       // MMA-issuing warps, at most
constexpr int GEMM_CODE_STAGE = GEMM_BM * 128;
constexpr int GEMM_SMEM_LIMIT = 227 * 1024;

// Shared-memory plan of the GEMM kernel (all offsets from a 1024-aligned base).
struct GemmSmem {
    int code_off, b_off, scale_off, meta_off, tok_off, shift_off, bar_off, misc_off, total;
};

__host__ __device__ inline int align_up(int v, int a) { return (v + a - 1) / a * a; }

__host__ __device__ inline int gemm_num_barriers(int n_c_stages, int n_a_slots, int n_b_stages) {
    // code full/empty, scale full/empty, A full/empty, B full/empty, D full/empty,
    // row-shift full/empty, one drain barrier per MMA warp
    return 2 * n_c_stages + 4 + 2 * n_a_slots + 2 * n_b_stages + 4 + 4 + GEMM_ISS_MAX;
}

// b_slot_bytes = b_unit * b_stage_bytes
__host__ __device__ inline GemmSmem gemm_smem_plan(int K, int E, int n_c_stages, int n_a_slots, int n_b_stages,
                                                    int b_slot_bytes) {
    GemmSmem s;
    s.code_off = 0;
    s.b_off = n_c_stages * GEMM_CODE_STAGE;
    s.scale_off = s.b_off + n_b_stages * b_slot_bytes;
    const int scale_bytes = align_up(GEMM_BM * (K / 32), 128);
    s.meta_off = s.scale_off + 2 * scale_bytes;
    s.tok_off = s.meta_off + 8 * (GEMM_NB_MAX / 2) * 4;         // per epilogue warp: one value per its columns
    s.shift_off = s.tok_off + GEMM_NB_MAX * 4;                  // producer's token list of the work item
    s.bar_off = s.shift_off + 2 * GEMM_BM * 4;
    s.misc_off = s.bar_off + align_up(gemm_num_barriers(n_c_stages, n_a_slots, n_b_stages) * 8, 16);
    // misc: tmem base, abort flag, then counts/offsets/tiles caches
    s.total = s.misc_off + 16 + 3 * (E + 1) * 4;
    s.total = align_up(s.total, 128) + 1024;  // slack for aligning the base
    return s;
}

}  // namespace moe
