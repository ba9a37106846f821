// Host-side helpers shared by the C ABI entry points: TMA descriptor encoding
// and the launch plan (ring depths, MMA warps, TMEM split) of the grouped GEMM.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>

#include "kernels.cuh"
#include "moe_b200.h"

namespace moe {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// u8 codes [E][R][K/2]: box {128 bytes, box_rows, 1}, 128-byte swizzle, zero fill out of range.
inline bool encode_codes(CUtensorMap *m, const void *codes, int E, int R, int K, int box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)(K / 2), (cuuint64_t)R, (cuuint64_t)E};
    const cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)R * (K / 2)};
    const cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(codes), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp16 K-blocked [cols/64][rows][64]: 3-D box {64, box_rows, box_kb}, 128-byte swizzle.
inline bool encode_f16_blocked(CUtensorMap *m, const void *base, int rows, int cols, int box_rows, int box_kb) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
    const cuuint64_t strides[2] = {128, (cuuint64_t)rows * 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_kb};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token rows per GEMM work item.  Decode-sized batches (T <= 64) use blocks of
// 16 rows: experts then rarely hold more than one block, and the small
// accumulators leave TMEM to the A slots; an expert with more tokens takes
// extra blocks whose weight re-reads hit L2.  Larger batches use the smallest
// multiple of 16 that holds every token (an expert receives each token at
// most once), capped at 256.
inline int token_block_rows(int T) {
    if (T <= 64) return 16;
    int nb = ((T > 0 ? T : 1) + 15) / 16 * 16;
    return nb < 256 ? nb : 256;
}

// Rows per B TMA box: the whole token block up to 64 rows (a TMA instruction
// holds its issuing thread ~100+ cycles, so fewer, larger boxes).  When one
// box holds the whole token block it also spans four 64-K blocks.
inline int b_box_rows(int nb_rows) { return nb_rows < 64 ? nb_rows : 64; }
inline int b_unit(int nb_rows) { return nb_rows <= 64 ? 4 : 1; }

// Shapes, ring depths, MMA warps and the TMEM split of one grouped GEMM
// launch for T tokens; fills everything of p except the pointers and the
// tensor maps.  Returns MOE_ERR_ARG when the plan does not fit.
inline int plan_gemm(GemmParams &p, int mode, int T, int top_k, int d, int F, int E, int P_max, int num_sms,
                     int *grid, int *smem) {
    p.nb_rows = token_block_rows(T);
    p.b_box_rows = b_box_rows(p.nb_rows);
    p.b_unit = b_unit(p.nb_rows);
    if (mode == MODE_UP) {
        p.K = d;
        p.R = 2 * F;
        p.MB = F / 64;
        p.out_ld = F;
    } else {
        p.K = F;
        p.R = d;
        p.MB = (d + GEMM_BM - 1) / GEMM_BM;
        p.out_ld = d;
    }
    p.F = F;
    p.E = E;
    p.b_stage_bytes = (p.nb_rows + p.b_box_rows - 1) / p.b_box_rows * p.b_box_rows * 128;
    p.b_rows_total = P_max;
    const int b_slot = p.b_unit * p.b_stage_bytes;
    // MMA warps: a tcgen05.mma holds its issuing thread ~120 cycles, so small
    // token blocks use up to three issuers (each its own accumulator)
    const int n_sub = p.K / GEMM_KA;
    const int n_chunks = (n_sub + 1) / 2;              // decoder chunks of two sub-stages per work item
    int ni = 256 / p.nb_rows;
    if (ni > GEMM_ISS_MAX) ni = GEMM_ISS_MAX;
    if (ni < 1) ni = 1;
    // decoder groups: three when several MMA warps share the work (small token
    // blocks, decode is the scarce resource), else two; never more groups than
    // chunks per work item, and never more MMA warps than groups, so every MMA
    // warp gets a chunk of every work item
    int ng = ni >= 2 ? 3 : 2;
    if (ng > n_chunks) ng = n_chunks;
    if (ni > ng) ni = ng;
    p.n_iss = ni;
    p.n_dec_groups = ng;
    p.n_d_bufs = (2 * ni * p.nb_rows <= 256) ? 2 : 1;
    // TMEM: A slots first, then the accumulators
    p.n_a_slots = (512 - p.n_d_bufs * ni * p.nb_rows) / 32;
    if (p.n_a_slots > GEMM_NA_MAX) p.n_a_slots = GEMM_NA_MAX;
    p.n_a_slots &= ~1;
    if (p.n_a_slots / 2 < p.n_dec_groups) return MOE_ERR_ARG;   // every decoder group owns a slot pair
    // shared memory: up to 8 code stages next to the B ring, then whatever is
    // left goes to the code ring
    const GemmSmem fixed = gemm_smem_plan(p.K, E, 0, p.n_a_slots, 0, b_slot);
    const int room = GEMM_SMEM_LIMIT - fixed.total - 8 * 2 * (GEMM_SC_MAX + 16);
    // B fills of 4 sub-stages are shared by two decoder/MMA pipelines and must
    // run well ahead of both: up to 8 of them (32 sub-stages); per-sub-stage
    // fills (large token blocks) up to 16
    int nbs = p.b_unit == 4 ? 8 : 16, sc = 8;
    const int nbs_min = p.b_unit == 4 ? 2 : 3;
    while (sc * GEMM_CODE_STAGE + nbs * b_slot > room && sc > 6) --sc;
    while (sc * GEMM_CODE_STAGE + nbs * b_slot > room && nbs > nbs_min) --nbs;
    while (sc * GEMM_CODE_STAGE + nbs * b_slot > room && sc > 4) --sc;
    while ((sc + 1) * GEMM_CODE_STAGE + nbs * b_slot <= room && sc < GEMM_SC_MAX) ++sc;
    if (sc * GEMM_CODE_STAGE + nbs * b_slot > room) return MOE_ERR_ARG;
    p.n_b_stages = nbs;
    p.n_c_stages = sc;
    const GemmSmem plan = gemm_smem_plan(p.K, E, p.n_c_stages, p.n_a_slots, p.n_b_stages, b_slot);
    if (plan.total > GEMM_SMEM_LIMIT) return MOE_ERR_ARG;
    *smem = plan.total;
    const long long P = (long long)T * top_k;
    const long long max_blocks = (P < E ? P : E) + P / p.nb_rows;
    const long long max_work = (long long)p.MB * max_blocks;
    int g = num_sms;
    if (max_work < g) g = (int)(max_work > 0 ? max_work : 1);
    *grid = g;
    return MOE_OK;
}

}  // namespace moe
