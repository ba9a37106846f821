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

// The driver's tensor-map encoder, looked up once per process (a function-local
// static: its initialisation is thread-safe, so first calls from several host
// threads do not race).
inline EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(f);
        return nullptr;
    }();
    return fn;
}

// E2M1 codes of W13 (u8 [E][2F][K/2]) for the gate/up GEMM, unpacked by TMA
// to one byte per element in shared memory.  A 5-D view whose box is 16 gate
// rows, their 16 linear rows, then the next group of 16 of each, four times:
// shared row 32q + l holds gate row 16q + l (l < 16) or linear row 16q + l - 16
// of the 64-row block, so each gate row and its linear partner land in one warp's
// TMEM lanes.  Only the first K_main (multiple of 128) columns are mapped.
inline bool encode_a_up(CUtensorMap *m, const void *codes, int E, int F, int K, int K_main) {
    EncodeTiledFn f = encode_fn();
    if (!f || K_main < 128) return false;
    const cuuint64_t row = (cuuint64_t)K / 2;
    const cuuint64_t dims[5] = {(cuuint64_t)K_main, 16, 2, (cuuint64_t)(F / 16), (cuuint64_t)E};
    const cuuint64_t strides[4] = {row, (cuuint64_t)F * row, 16 * row, 2 * (cuuint64_t)F * row};
    const cuuint32_t box[5] = {128, 16, 2, 4, 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 5, const_cast<void *>(codes), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E2M1 codes of W2 (u8 [E][d][K/2]) for the down GEMM: box {128, 128 rows, 1};
// rows past d read as zero.
inline bool encode_a_down(CUtensorMap *m, const void *codes, int E, int d, int K, int K_main) {
    EncodeTiledFn f = encode_fn();
    if (!f || K_main < 128) return false;
    const cuuint64_t row = (cuuint64_t)K / 2;
    const cuuint64_t dims[3] = {(cuuint64_t)K_main, (cuuint64_t)d, (cuuint64_t)E};
    const cuuint64_t strides[2] = {row, (cuuint64_t)d * row};
    const cuuint32_t box[3] = {128, 128, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void *>(codes), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 B operand u8 [3 planes][rows][Kpad] (hi, lo and lo2 planes, each `rows`
// rows): a 3-D view {Kpad, rows, 3} whose box {128 bytes, box_rows, box_planes}
// brings a token block's rows of box_planes consecutive planes in one copy,
// plane by plane in shared memory; 128-byte swizzle, zero fill past the last row
// and past the last plane.
inline bool encode_bq(CUtensorMap *m, const void *base, int rows, int Kpad, int box_rows, int box_planes) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)Kpad, (cuuint64_t)rows, 3};
    const cuuint64_t strides[2] = {(cuuint64_t)Kpad, (cuuint64_t)rows * Kpad};
    const cuuint32_t box[3] = {128, (cuuint32_t)box_rows, (cuuint32_t)box_planes};
    const cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int round_up_128(int v) { return (v + 127) / 128 * 128; }

// Token rows per GEMM work item.  Decode-sized batches (T <= 64) use blocks of
// 16 rows: their three terms stack into one MMA of N = 48; experts then rarely
// hold more than one block, and an expert with more tokens takes extra blocks
// whose weight re-reads hit L2.  Larger batches use the smallest multiple of 16
// that holds every token (an expert receives each token at most once), capped
// at GEMM_NB_MAX.
inline int token_block_rows(int T) {
    if (T <= 64) return 16;
    int nb = ((T > 0 ? T : 1) + 15) / 16 * 16;
    return nb < GEMM_NB_MAX ? nb : GEMM_NB_MAX;
}

// Shapes, ring depth and TMEM split of one grouped GEMM launch for T tokens;
// fills everything of p except the pointers and the tensor maps.  Returns
// MOE_ERR_ARG when the plan does not fit.
inline int plan_gemm(GemmParams &p, int mode, int T, int top_k, int d, int F, int E, int P_max, int num_sms,
                     int *grid, int *smem) {
    p.nb_rows = token_block_rows(T);
    // small token blocks: one MMA over the hi, lo and lo2 rows together (N = 3 nb_rows, rounded up to 16)
    p.stacked = p.nb_rows <= 64 ? 1 : 0;
    if (mode == MODE_UP) {
        p.K = d;
        p.R = 2 * F;
        p.MB = F / 64;
    } else {
        p.K = F;
        p.R = d;
        p.MB = (d + GEMM_BM - 1) / GEMM_BM;
    }
    p.K_main = p.K / GEMM_KS * GEMM_KS;
    p.F = F;
    p.E = E;
    p.P_max = P_max;
    p.Kf = round_up_128(F);
    // per-item scale factors (and two MMA warps) when a stacked block's item
    // regions fit in TMEM next to the two MMA warps' accumulators
    const int n_st = (p.K + GEMM_KS - 1) / GEMM_KS;
    // (an item region's B group holds the scale words of at most 128 stacked rows)
    p.sf_item = p.stacked && 3 * p.nb_rows <= 128 && n_st <= GEMM_SFI_STAGES_MAX &&
                gemm_tmem_cols_item(p.nb_rows, p.stacked, n_st) <= 512 ? 1 : 0;
    auto fits = [&](int ns) {
        return gemm_smem_plan(p.K, E, p.nb_rows, p.stacked, ns, p.sf_item).total <= GEMM_SMEM_LIMIT &&
               (p.sf_item || gemm_tmem_cols(p.nb_rows, p.stacked, ns) <= 512);
    };
    // as many stages as shared memory (and, per stage, TMEM) hold
    int ns = GEMM_STAGES_MAX;
    while (ns > 2 && !fits(ns)) --ns;
    if (!fits(ns)) return MOE_ERR_ARG;
    p.n_stages = ns;
    *smem = gemm_smem_plan(p.K, E, p.nb_rows, p.stacked, ns, p.sf_item).total;
    const long long P = (long long)T * top_k;
    const long long max_blocks = (P < E ? P : E) + P / p.nb_rows;
    const long long max_work = (long long)p.MB * max_blocks;
    int g = num_sms;
    if (max_work < g) g = (int)(max_work > 0 ? max_work : 1);
    *grid = g;
    return MOE_OK;
}

}  // namespace moe
