// Kernel parameter blocks and launch-side constants shared by api.cu and the
// kernel sources.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace moe {

// Launch `kernel` on `s` with programmatic stream serialization: it may begin
// (and run its prologue) while the previous kernel of the stream finishes;
// the kernels call pdl_wait() before reading anything a predecessor wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Error bits of the device error word.
enum : unsigned int {
    ERR_WAIT_UP = 1u,      // a bounded wait ran out in the gate/up GEMM
    ERR_WAIT_DOWN = 2u,    // ... in the down GEMM
    ERR_WAIT_SELFTEST = 4u,
    ERR_ROUTING = 8u,      // an expert index out of range reached the grouping
    ERR_WAIT_ROUTE = 16u   // the grid barrier of the decode-sized route + group launch ran out
};

struct RouteParams {
    const uint16_t *x;          // bf16 [T, d]
    const uint16_t *norm_scale; // bf16 [d]
    const uint16_t *router_w;   // bf16 [E, d]
    const float *router_b;      // fp32 [E]
    int T, d, E, k;
    float eps;
    float *xn;                  // fp32 [T, d] normalised tokens
    int *topk_idx;              // [T, k]
    float *topk_w;              // [T, k]
    float *logits;              // fp32 [T, E] (decode-sized path: the CTAs' share of each token's logits)
    unsigned int *tok_done;     // [T] CTAs finished per token (decode-sized path); zero between calls
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
    // the expert-sorted E4M3 terms of the normalised tokens (gate/up B operand)
    const float *xn;            // fp32 [T, d]
    uint8_t *xq;                // [3][P_max][Kd]: hi, lo, lo2 planes
    unsigned int *h_ready;      // the fused decode GEMM's per-token-block counters, zeroed by the
    int n_h_ready;              //   decode-sized route + group launch (NULL: none)
    uint32_t *xsf;              // [Kd/128][2][P_max]: scales of the hi (also lo2) and lo planes
    int P_max, d, Kd;
};

// Grouped block-scaled GEMM over (expert, 128-row weight block, token block)
// work items: MXFP4 weights (E2M1 codes, E8M0 block scales) times the
// activations held as three E4M3 terms per 32-element block with exponent s:
//   hi  = e4m3(v / 2^s),  lo = e4m3((v - hi 2^s) / 2^(s-4)),
//   lo2 = e4m3((v - hi 2^s - lo 2^(s-4)) / 2^s)
// (hi and lo keep about 8 significant bits of v, the three together about 12;
// lo2 shares hi's scale byte, so an MMA over lo2 rows reads hi's scale
// column).  fp32 accumulation in TMEM.  Stacked token blocks (decode-sized)
// always use all three terms in one MMA; large blocks use hi + lo, and add a
// pass over lo2 for work items whose weights reach E8M0 byte LO2_SCALE_MIN.
// MODE_UP: rows are the gate/linear pairs of W13, epilogue is the clamped
// SwiGLU, written as the down GEMM's B.  MODE_DOWN: rows are W2's, epilogue
// writes the routing-weighted expert output rows.
// MODE_FFN: both GEMMs of a decode-sized batch in one persistent launch -- the
// gate/up items, then the down items; a down item waits until every gate/up
// item of its token block has written its h rows (a counter per token block).
enum { MODE_UP = 0, MODE_DOWN = 1, MODE_FFN = 2 };

struct GemmParams {
    CUtensorMap map_a;          // E2M1 codes, 16 x 4-bit per 16 bytes in shared memory (unpacked TMA type);
                                //   UP: 5-D {K_main, 16 rows, 2 halves, F/16 groups, E}, box {128, 16, 2, 4, 1}
                                //   DOWN: 3-D {K_main, d, E}, box {128, 128, 1}
    CUtensorMap map_b;          // u8 [3][P_max][Kpad] E4M3 hi, lo, lo2 planes; box {128, nb_rows, 3 stacked / 2}
    const uint8_t *codes;       // u8 [E][R][K/2] (the K tail is read directly)
    const uint8_t *scales;      // u8 [E][R][K/32]
    const uint16_t *bias;       // bf16 [E][R]
    const uint32_t *b_sf;       // [Kpad/128][2][P_max] words: E8M0 scales of 4 consecutive 32-blocks of B
    int K;                      // reduction length (multiple of 64)
    int K_main;                 // K rounded down to a multiple of 128 (TMA-loaded part)
    int R;                      // rows per expert: 2F (UP) or d (DOWN)
    int F;                      // d_ff (UP: gate rows [0,F), linear rows [F,2F))
    int E;
    int MB;                     // weight blocks per expert: F/64 (UP) or ceil(d/128) (DOWN)
    int nb_rows;                // token rows per work item (multiple of 16, <= GEMM_NB_MAX)
    int stacked;                // 1: one MMA covers the hi, lo and lo2 rows (N = 3 nb_rows); 0: one MMA per term
    int n_stages;               // shared-memory ring depth (and TMEM scale-factor ring depth when !sf_item)
    int sf_item;                // 1: a work item's scale factors are written to TMEM once, before its first
                                //    stage, and two MMA warps take alternate stages (decode-sized blocks);
                                // 0: scale factors per stage in a TMEM ring, one MMA warp
    int P_max;                  // rows of each B plane
    const int *counts, *offsets, *tiles;
    const int *row_token;       // [P]
    const float *row_w;         // [P]
    // UP output: the down GEMM's B (three E4M3 planes [3][P_max][Kf]) and its scales
    uint8_t *h_q;
    uint8_t *h_sf;              // bytes of [Kf/128][2][P_max] words
    int Kf;                     // F rounded up to 128
    // Large blocks: the pass count of each work item's weight block, u8 [E][MB]: 1, or 2 with a
    // pass over the lo2 term (weights reaching LO2_SCALE_MIN); NULL: one pass.  Stacked blocks
    // carry all three terms in one pass.
    const uint8_t *item_pass;
    int item_pass_stride;       // bytes per expert in item_pass
    // UP, large blocks: the down GEMM's pass counts u8 [E][DOWN_PASS_STRIDE]; h gets its lo2
    // plane for the experts with a two-pass down item (stacked blocks always write it)
    const uint8_t *down_pass;
    int MB_down;
    // DOWN output: fp32 weighted rows [P][d]
    float *out_rows;
    unsigned int *err;
    unsigned long long wait_limit_ns;
    // MODE_FFN: per token block (index tiles[e] + block), the gate/up epilogue warps that have
    // written their h rows; a down item of the block starts at h_target (8 x gate/up weight blocks)
    unsigned int *h_ready;
    unsigned int h_target;
};

constexpr int GEMM_THREADS = 512;     // 16 warps
constexpr int GEMM_BM = 128;          // weight rows per work item (TMEM lanes)
constexpr int GEMM_KS = 128;          // K elements per stage (4 MMAs of K = 32)
constexpr int GEMM_NB_MAX = 192;      // token rows per work item, at most
constexpr int GEMM_STAGES_MAX = 12;
constexpr int GEMM_A_STAGE = GEMM_BM * 128;   // unpacked E2M1: one byte per element in shared memory
constexpr int GEMM_SF_COLS = 24;      // TMEM columns per scale-factor slot: A at +0, B hi at +8, B lo at +16
// Large token blocks add a pass over the third activation term (lo2) to the work
// items whose weight rows hold an E8M0 byte of at least this (weights of
// magnitude 3 or more: 6 * 2^-1).  Below it two terms keep the block well inside
// its tolerance; above it the pre-activations grow large enough that two-term
// rounding of the activations moves the clamped SwiGLU's output.
constexpr int LO2_SCALE_MIN = 126;
// Row stride (bytes) of the down GEMM's pass table: at least its weight blocks per expert
// (ceil(d_model / 128) <= 48), so that a warp reads an expert's row in one load.
constexpr int DOWN_PASS_STRIDE = 64;
constexpr int GEMM_SMEM_LIMIT = 227 * 1024;

// Shared-memory plan of the GEMM kernel (all offsets from a 1024-aligned base).
struct GemmSmem {
    int a_off, b_off, scale_off, amax_off, meta_off, bsf_off, bar_off, misc_off, total;
};

// Per-item mode: the B scale words of one work item, staged in shared memory
// for the scale-factor warps ([stage][4 columns][32 lanes] words; a fixed
// stride of four columns -- a stride by the block's column count measured
// 12% slower on the decode-sized down GEMM).
constexpr int GEMM_SFI_STAGES_MAX = 24;
constexpr int GEMM_SFI_BSF_BYTES = GEMM_SFI_STAGES_MAX * 4 * 32 * 4;

__host__ __device__ inline int align_up(int v, int a) { return (v + a - 1) / a * a; }

__host__ __device__ inline int gemm_num_barriers(int n_stages) {
    // stage full/empty [NS], A-scale full/empty [2], D full [2 MMA warps][2], D empty [2],
    // drain [2], epilogue exchange [2][2], item scale factors full/empty [2], staged B words full/empty,
    return 2 * n_stages + 4 + 4 + 2 + 2 + 4 + 4 + 2;
}

// B ring slot: the token block's hi, lo and lo2 rows (stacked) or two planes (hi and lo, or lo2
// and an empty plane in a lo2 pass)
__host__ __device__ inline int gemm_b_planes(int stacked) { return stacked ? 3 : 2; }
__host__ __device__ inline int gemm_b_stage_bytes(int nb_rows, int stacked) {
    return gemm_b_planes(stacked) * nb_rows * 128;
}

__host__ __device__ inline GemmSmem gemm_smem_plan(int K, int E, int nb_rows, int stacked, int n_stages,
                                                   int sf_item) {
    GemmSmem s;
    s.a_off = 0;
    s.b_off = n_stages * GEMM_A_STAGE;
    s.scale_off = s.b_off + n_stages * gemm_b_stage_bytes(nb_rows, stacked);
    const int scale_bytes = align_up(GEMM_BM * (K / 32), 128);
    // A scale bytes: double-buffered per-stage mode (bulk copies one item ahead), one buffer per-item mode
    s.amax_off = s.scale_off + (sf_item ? 1 : 2) * scale_bytes;
    s.meta_off = s.amax_off + 2 * 2 * 4 * 16 * 4;                 // [2 groups][2 parities][4 warps][16 columns] fp32
    s.bsf_off = s.meta_off + align_up(8 * nb_rows * 4, 16);        // per epilogue warp: one value per column
    s.bar_off = s.bsf_off + (sf_item ? GEMM_SFI_BSF_BYTES : 0);
    s.misc_off = s.bar_off + align_up(gemm_num_barriers(n_stages) * 8, 16);
    // misc: tmem base, abort flag, then counts/offsets/tiles caches
    s.total = s.misc_off + 16 + 3 * (E + 1) * 4;
    s.total = align_up(s.total, 128) + 1024;  // slack for aligning the base
    return s;
}

// TMEM columns of the plan.  Per-stage mode: accumulators (2 buffers), then the
// ring of scale-factor slots.  Per-item mode: accumulators [2 MMA warps] (one
// buffer each), then two item regions of 8 columns per stage (A at +0, B at +4).
constexpr int GEMM_SFI_COLS = 8;
__host__ __device__ inline int gemm_d_cols(int nb_rows, int stacked) { return stacked ? 3 * nb_rows : nb_rows; }
__host__ __device__ inline int gemm_tmem_cols(int nb_rows, int stacked, int n_stages) {
    return 2 * gemm_d_cols(nb_rows, stacked) + GEMM_SF_COLS * n_stages;
}
__host__ __device__ inline int gemm_tmem_cols_item(int nb_rows, int stacked, int n_st) {
    return 2 * gemm_d_cols(nb_rows, stacked) + 2 * GEMM_SFI_COLS * n_st;
}

}  // namespace moe
