// Grouped MXFP4 expert GEMMs of the MoE block on sm_100a: block-scaled
// tcgen05 MMAs (kind::mxf8f6f4, E2M1 weights x E4M3 activations, E8M0 block
// scales) with TMA-fed shared-memory rings and fp32 accumulators in TMEM.
//
// One persistent CTA per SM walks the work items (expert e, 128-row weight
// block, block of up to GEMM_NB_MAX tokens routed to e).  Per 128-K stage:
//   A (weights, M = 128 rows): the packed E2M1 codes go from HBM to shared
//     memory by TMA with the unpacked 4-bit type (16 codes per 16 bytes, the
//     operand layout of the block-scaled MMA) and a 128-byte swizzle.  No
//     thread touches a weight element: the tensor core applies the E8M0 block
//     scales itself ("MXFP4": 32 elements share one power of two, pnsm.cn
//     overview sections 1 and 4).  A K tail of 64 (K = 2880 = 22.5 x 128) is
//     loaded by the A producer with plain loads at the item's start and written
//     into its stage's slot in the unpacked layout.
//   B (activations, N = tokens): E4M3 terms per 32-element block with E8M0
//     scale s chosen so the block maximum fits 448: hi = e4m3(v / 2^s),
//     lo = e4m3((v - hi 2^s) / 2^(s-4)) and lo2 = e4m3((v - hi 2^s - lo
//     2^(s-4)) / 2^s).  hi + lo keep about 8 significant bits of every element
//     (the precision of bf16), the three terms about 12 (that of the fp16
//     normalised tokens).  lo2 uses hi's scale byte, so its MMA reads hi's
//     scale column.  Small (decode-sized) blocks stack a token block's hi, lo
//     and lo2 rows in one MMA (N = 3 x rows, the epilogue adds the thirds).
//     Large blocks run one MMA over hi and one over lo per K block into the
//     same accumulator; a work item whose weights reach the E8M0 byte
//     LO2_SCALE_MIN then takes a second pass over K with the lo2 rows.
//   Scale factors: the scale-factor warps write A's and B's E8M0 bytes into
//     TMEM, one 32-bit column per 32 rows, the byte index being the 32-block
//     within the stage, replicated in all four lane quarters (the layout the
//     block-scaled MMA reads): per stage into a slot of a ring, or per work
//     item into one of two item regions.
// Gate/up epilogue: z = D + b13, clamped SwiGLU
//   h = min(g,7) * sigmoid(1.702 min(g,7)) * (clamp(u,-7,7) + 1)
//   ("gpt-oss-20B" hub page, section 3.3).  Each 128-row weight block holds 64
//   gate rows and their 64 linear rows, interleaved in groups of 16 by the
//   tensor map, so each pair meets in one warp.  h is written directly as the
//   down GEMM's B (three E4M3 planes): the block maxima over 32 consecutive h
//   rows are exchanged between the two warps holding them.
// Down epilogue: o = w_token * (D + b2) written to the pair's expert-sorted
//   row; the combine kernel adds a token's rows to its residual (weighted
//   combine, "gpt-oss-20B" page section 3.4; pnsm.cn overview 2.2).
// MODE_FFN (decode-sized batches, d_model == d_ff): one launch walks the
//   gate/up items, then the down items, with the same per-item code as the two
//   separate launches.  A gate/up item's eight epilogue warps each count their
//   h stores into the token block's counter once they are fenced; a down item's
//   B producer and scale-factor warps wait (bounded) until the counter reaches
//   eight per gate/up weight block, and the B producer then orders its TMA reads
//   of h after that acquire (a proxy fence).  Every CTA takes its gate/up items
//   before its down items and only down items wait, on gate/up items, so every
//   wait ends once the grid is resident.
//
// Warp roles (512 threads): 0 TMA producer of A (weights), 3 TMA producer of
// B (activations), 1 MMA issue, 2 TMEM allocation and (per-item scale factors)
// the second MMA warp, 4-7 scale-factor warps (one per TMEM lane quarter),
// 8-11 and 12-15 two epilogue groups taking 16-column chunks in turn.
// Large blocks: every role reads a work item's pass count (one, or two with the
// lo2 pass) from a table that pass_plan_kernel writes from the weights' scale
// bytes before the gate/up GEMM.
// Producers and MMA run as whole converged warps, one elected lane issuing.
// Every mbarrier wait is bounded (WaitCtl); when one runs out the CTA stops
// issuing work, drains its copies and MMAs in flight, frees TMEM and returns
// with the error latched.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int SF_PD = 4;        // stages of B scale words the scale-factor warps load ahead
constexpr int SF_WORDS = 12;    // B scale words per lane and stage, at most (6 columns x hi/lo)

struct Work {
    int e, mb, p0, n_valid, n_mma;
    int blk;        // the token block's index over all experts (tiles[e] + block)
    bool up;        // a gate/up item (always in MODE_UP launches, never in MODE_DOWN ones)
};

__device__ __forceinline__ void work_of(int w, const int *tiles_s, const int *counts_s, const int *offsets_s, int E,
                                        int MB, int nb_rows, int P_max, Work &t) {
    // the last expert e with MB * tiles[e] <= w has at least one token block
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (MB * tiles_s[mid] <= w) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int local = w - MB * tiles_s[e];
    const int nblk = tiles_s[e + 1] - tiles_s[e];
    t.e = e;
    t.mb = local / nblk;
    const int nb = local - t.mb * nblk;
    t.blk = tiles_s[e] + nb;
    t.p0 = offsets_s[e] + nb * nb_rows;
    t.n_valid = min(nb_rows, counts_s[e] - nb * nb_rows);
    // never past the row buffers, even for routing arrays that do not match (the down
    // GEMM reads them before its dependency wait; see the kernel's prologue)
    t.n_valid = max(0, min(t.n_valid, P_max - t.p0));
    t.n_mma = max(16, (t.n_valid + 15) & ~15);     // a valid MMA width (16..nb_rows) in any case
}

__device__ __forceinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity, unsigned long long limit_ns) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - start > limit_ns) return;
    }
}

// Wait for the `n_issued` most recent fills of a ring of `n_slots` full
// barriers (fill i went to slot i % n_slots with phase parity (i / n_slots) & 1).
__device__ __forceinline__ void drain_ring(uint64_t *full, int n_slots, long long n_issued,
                                           unsigned long long limit_ns) {
    for (long long i = n_issued - 1; i >= 0 && i >= n_issued - n_slots; --i)
        mbar_wait_drain(&full[i % n_slots], (uint32_t)((i / n_slots) & 1), limit_ns);
}

// Passes over K of work item t: 2 (the hi and lo terms, then the lo2 term) where
// the pass table says so, else 1.
__device__ __forceinline__ int item_passes(const GemmParams &p, const Work &t) {
    return p.item_pass ? (int)__ldg(p.item_pass + (size_t)t.e * p.item_pass_stride + t.mb) : 1;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Source row (0..127) in the work item's scale buffer of tile row r (the A
// row in shared memory and TMEM lane r).  Gate/up: the buffer holds the 64 gate
// rows then the 64 linear rows; tile row 32q + l is gate row 16q + l (l < 16) or
// linear row 16q + l - 16.
__device__ __forceinline__ int tile_scale_row(bool up, int r) {
    if (up) {
        const int q = r >> 5, l = r & 31;
        return l < 16 ? 16 * q + l : 64 + 16 * q + (l - 16);
    }
    return r;
}

// Weight row of tile row r in the expert's row space (gate/up: [0, 2F); down: [0, d)).
__device__ __forceinline__ int tile_weight_row(bool up, int r, int mb, int F) {
    if (up) {
        const int q = r >> 5, l = r & 31;
        return l < 16 ? mb * 64 + 16 * q + l : F + mb * 64 + 16 * q + (l - 16);
    }
    return mb * GEMM_BM + r;
}

// Bounded wait until a counter another CTA releases reaches `target` (as mbar_wait:
// false when the CTA has aborted or the wait ran out, which aborts the CTA).
__device__ __forceinline__ bool wait_count(const unsigned int *ctr, unsigned int target, const WaitCtl &w) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    const uint64_t start = globaltimer_ns();
    for (;;) {
        __nanosleep(128);
        if (ld_acquire_gpu(ctr) >= target) return true;
        if (*w.abort) return false;
        if (globaltimer_ns() - start > w.limit_ns) {
            *w.abort = 1;
            atomicOr(w.err, w.err_bit);
            return false;
        }
    }
}

// p: the launch's GEMM (MODE_UP, MODE_DOWN) or, in MODE_FFN, the gate/up GEMM; p2: the down
// GEMM in MODE_FFN (the same as p otherwise).  MODE_FFN needs d_model == d_ff (one K for both).
template <int MODE, bool SFI>
__global__ void __launch_bounds__(GEMM_THREADS, 1) expert_gemm_kernel(const __grid_constant__ GemmParams p,
                                                                      const __grid_constant__ GemmParams p2) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = p.n_stages;
    const int NB = p.nb_rows;
    const GemmSmem plan = gemm_smem_plan(p.K, p.E, NB, p.stacked, NS, SFI ? 1 : 0);
    uint8_t *a_ring = smem + plan.a_off;
    uint8_t *b_ring = smem + plan.b_off;
    const int b_stage = gemm_b_stage_bytes(NB, p.stacked);
    uint8_t *scale_buf = smem + plan.scale_off;
    const int KB32 = p.K / 32;
    const int scale_bytes = align_up(GEMM_BM * KB32, 128);
    float *amax_s = reinterpret_cast<float *>(smem + plan.amax_off);   // [2 groups][2 parities][4 warps][16 columns]
    float *meta_val = reinterpret_cast<float *>(smem + plan.meta_off);  // [8 warps][NB]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + plan.bar_off);
    uint64_t *full = bars;
    uint64_t *empty = full + NS;
    uint64_t *s_full = empty + NS;          // [2] A scale bytes of a work item in shared memory
    uint64_t *s_empty = s_full + 2;
    uint64_t *d_full = s_empty + 2;         // [2 MMA warps][2 accumulator buffers]
    uint64_t *d_empty = d_full + 4;         // [2]
    uint64_t *drain_bar = d_empty + 2;      // [2 MMA warps]
    uint64_t *ex_bar = drain_bar + 2;       // [2 groups][2 parities]
    uint64_t *f_full = ex_bar + 4;          // [2] a work item's scale factors in TMEM (per-item mode)
    uint64_t *f_empty = f_full + 2;
    uint64_t *bw_full = f_empty + 2;        // the item's B scale words are staged (per-item mode)
    uint64_t *bw_empty = bw_full + 1;       // ... and have been read by all four scale-factor warps
    uint32_t *bw_s = reinterpret_cast<uint32_t *>(smem + plan.bsf_off);   // [stage][4][32]
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + plan.misc_off);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + plan.misc_off + 4);
    int *counts_s = reinterpret_cast<int *>(smem + plan.misc_off + 16);
    int *offsets_s = counts_s + (p.E + 1);
    int *tiles_s = offsets_s + (p.E + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_st = (p.K + GEMM_KS - 1) / GEMM_KS;     // stages per work item
    const int n_main = p.K_main / GEMM_KS;              // stages loaded by TMA; a last one past them is the K tail
    const int d_cols = gemm_d_cols(NB, p.stacked);
    // MMA warps: two taking alternate stages in per-item mode (the second only
    // when an item has more than one stage), one otherwise
    const int n_mma_warps = SFI && n_st > 1 ? 2 : 1;
    // accumulator buffers per MMA warp: two (the epilogue drains one while the MMAs
    // fill the other), one in per-item mode, where the two MMA warps' accumulators
    // and the two item regions of scale factors fill TMEM
    constexpr int n_dbuf = SFI ? 1 : 2;
    // TMEM columns: accumulators first, then the scale factors
    const uint32_t sf_col0 = (uint32_t)(2 * d_cols);
    const int sfi_cols = GEMM_SFI_COLS * n_st;           // one item region (per-item mode)

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            // the two producers' arrivals (+ the four scale-factor warps per stage)
            mbar_init(&full[i], SFI ? 2 : 2 + 4);
            mbar_init(&empty[i], 1);      // MMA commit
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 4);
            mbar_init(&d_empty[i], 8);    // every epilogue warp
            mbar_init(&drain_bar[i], 1);
            mbar_init(&f_full[i], 4);     // the four scale-factor warps
            mbar_init(&f_empty[i], n_mma_warps);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&d_full[i], 1);
            mbar_init(&ex_bar[i], 4);     // the four warps of an epilogue group
        }
        mbar_init(bw_full, 4);            // the four scale-factor warps
        mbar_init(bw_empty, 4);
        *abort_s = 0;
        fence_barrier_init();
    }
    if (warp == 2) {
        tmem_alloc(tmem_base_s, 512);
        tmem_relinquish();
    }
    // The routing arrays come from the group kernel and the B operand from the
    // kernel before this one.  The gate/up GEMM follows the group kernel and
    // waits for it here.  The down GEMM follows the gate/up GEMM, which starts
    // its dependents only once it has itself waited for the group kernel: so
    // the down GEMM reads the routing arrays (from L2) at once, and only its
    // B producer and the loads of B scale words wait for the gate/up GEMM.
    // Its weight copies and weight scales start while the gate/up GEMM's last
    // CTAs finish.
    if constexpr (MODE == MODE_UP || MODE == MODE_FFN) pdl_wait();
    pdl_trigger();
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
        counts_s[i] = i < p.E ? __ldcg(p.counts + i) : 0;
        offsets_s[i] = __ldcg(p.offsets + i);
        tiles_s[i] = __ldcg(p.tiles + i);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    // work items: MODE_FFN runs the gate/up items [0, W_up), then the down items
    const GemmParams &pd = MODE == MODE_FFN ? p2 : p;    // the down items' GEMM
    const int W_up = p.MB * tiles_s[p.E];
    const int total = MODE == MODE_FFN ? W_up + pd.MB * tiles_s[p.E] : W_up;
    auto item_of = [&](int w, Work &t) {
        const bool up = MODE == MODE_FFN ? w < W_up : MODE == MODE_UP;
        const int wl = MODE == MODE_FFN && !up ? w - W_up : w;
        work_of(wl, tiles_s, counts_s, offsets_s, p.E, up ? p.MB : pd.MB, NB, p.P_max, t);
        t.up = up;
    };
    auto gp_of = [&](const Work &t) -> const GemmParams & { return t.up ? p : pd; };
    const WaitCtl wc{abort_s, p.err, MODE == MODE_DOWN ? (unsigned)ERR_WAIT_DOWN : (unsigned)ERR_WAIT_UP,
                     p.wait_limit_ns};

    if (warp == 0) {
        // ------------------------------------------------- A producer (weights)
        // Per work item (per-stage mode) the 128 rows' E8M0 bytes (one or two
        // untiled bulk copies), issued one item ahead so the scale-factor warps
        // can prepare an item while the MMAs work on the one before.  Per stage one
        // TMA box of E2M1 codes (128 rows x 128 K), the item's K stages once per
        // pass.  The K tail (K not
        // a multiple of 128) is loaded at the start of the item, four rows per
        // lane, and written into its stage's slot here.
        if (lane == 0 && n_main > 0) {
            tma_prefetch_desc(&p.map_a);
            if (MODE == MODE_FFN) tma_prefetch_desc(&p2.map_a);
        }
        int slot = 0, sb = 0;
        uint32_t ph = 0, sph = 0;
        long long issued = 0, s_issued = 0;
        bool ok = true;
        auto load_scales = [&](const Work &t) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(&s_empty[sb], sph ^ 1, wc))) return false;
            uint8_t *sdst = scale_buf + sb * scale_bytes;
            if (MODE == MODE_UP) {
                const int j0 = t.mb * 64;
                const uint32_t bytes = 64u * KB32;
                mbar_arrive_expect_tx_w(&s_full[sb], 2 * bytes);
                bulk_load_w(sdst, p.scales + ((size_t)t.e * p.R + j0) * KB32, bytes, &s_full[sb]);
                bulk_load_w(sdst + bytes, p.scales + ((size_t)t.e * p.R + p.F + j0) * KB32, bytes, &s_full[sb]);
            } else {
                const int m0 = t.mb * GEMM_BM;
                const uint32_t bytes = (uint32_t)min(GEMM_BM, p.R - m0) * KB32;
                mbar_arrive_expect_tx_w(&s_full[sb], bytes);
                bulk_load_w(sdst, p.scales + ((size_t)t.e * p.R + m0) * KB32, bytes, &s_full[sb]);
            }
            ++s_issued;
            if (++sb == 2) { sb = 0; sph ^= 1; }
            return true;
        };
        Work t;
        if (blockIdx.x < total) {
            item_of(blockIdx.x, t);
            if constexpr (!SFI) ok = load_scales(t);     // per-item mode: the scale-factor warps load them
        }
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            uint4 tail[8];                   // the item's K tail codes (rows lane + 32j)
            auto load_tail = [&]() {
                const GemmParams &q = gp_of(t);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int wrow = tile_weight_row(t.up, lane + 32 * j, t.mb, p.F);
                    tail[2 * j] = tail[2 * j + 1] = make_uint4(0, 0, 0, 0);
                    if (wrow < q.R) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            q.codes + ((size_t)t.e * q.R + wrow) * (p.K / 2) + p.K_main / 2);
                        tail[2 * j] = __ldg(src);
                        tail[2 * j + 1] = __ldg(src + 1);
                    }
                }
            };
            // the K tail codes, loaded at the start of the item so that the tail stage
            // does not wait on global memory
            if (n_st > n_main) load_tail();
            Work tn;
            const bool has_next = w + (int)gridDim.x < total;
            if (has_next) {
                item_of(w + gridDim.x, tn);
                if constexpr (!SFI) {
                    if (!load_scales(tn)) { ok = false; break; }
                }
            }
            // one K stage of A into the next ring slot
            auto issue_a = [&](int st) -> bool {
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[slot], ph ^ 1, wc))) return false;
                uint8_t *adst = a_ring + slot * GEMM_A_STAGE;
                if (st < n_main) {
                    // the unpacked-type TMA counts the packed bytes: 128 rows x 64
                    mbar_arrive_expect_tx_w(&full[slot], 128u * 64u);
                    if (t.up)
                        tma_load_5d_w(adst, &p.map_a, &full[slot], st * GEMM_KS, 0, 0, 4 * t.mb, t.e);
                    else
                        tma_load_3d_w(adst, &pd.map_a, &full[slot], st * GEMM_KS, t.mb * GEMM_BM, t.e);
                } else {
                    // K tail of rows lane + 32j: 2 x 16 code bytes -> the first four
                    // 16-byte units of the row (8 code bytes each, the rest zero),
                    // 128-byte swizzle
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int r = lane + 32 * j;
                        uint8_t *row = adst + r * 128;
                        const int sw = r & 7;
                        const uint4 c0 = tail[2 * j], c1 = tail[2 * j + 1];
                        *reinterpret_cast<uint4 *>(row + ((0 ^ sw) << 4)) = make_uint4(c0.x, c0.y, 0, 0);
                        *reinterpret_cast<uint4 *>(row + ((1 ^ sw) << 4)) = make_uint4(c0.z, c0.w, 0, 0);
                        *reinterpret_cast<uint4 *>(row + ((2 ^ sw) << 4)) = make_uint4(c1.x, c1.y, 0, 0);
                        *reinterpret_cast<uint4 *>(row + ((3 ^ sw) << 4)) = make_uint4(c1.z, c1.w, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    mbar_arrive_w(&full[slot]);
                }
                ++issued;
                if (++slot == NS) { slot = 0; ph ^= 1; }
                return true;
            };
            for (int st = 0; st < n_st; ++st) {
                if (!issue_a(st)) { ok = false; break; }
            }
            if constexpr (!SFI) {     // the lo2 pass: the item's K stages once more
                if (ok && item_passes(p, t) > 1) {
                    for (int st = 0; st < n_st; ++st) {
                        if (!issue_a(st)) { ok = false; break; }
                    }
                }
            }
            if (!ok) break;
            t = tn;
        }
        if (!ok) {
            drain_ring(full, NS, issued, p.wait_limit_ns);
            drain_ring(s_full, 2, s_issued, p.wait_limit_ns);
        }
    } else if (warp == 3) {
        // --------------------------------------------- B producer (activations)
        // Per stage one TMA box: the token block's rows of two planes (hi, lo) or,
        // stacked, of all three (hi, lo, lo2); in a lo2 pass the box starts at the
        // lo2 plane (the plane after it lies outside the map and reads as zeros).
        if (lane == 0) {
            tma_prefetch_desc(&p.map_b);
            if (MODE == MODE_FFN) tma_prefetch_desc(&p2.map_b);
        }
        if constexpr (MODE == MODE_DOWN) pdl_wait();     // h comes from the gate/up GEMM
        int slot = 0;
        uint32_t ph = 0;
        long long issued = 0;
        bool ok = true;
        const uint32_t b_bytes = (uint32_t)b_stage;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            Work t;
            item_of(w, t);
            if (MODE == MODE_FFN && !t.up) {
                // a down item: its token block's h rows, written by the gate/up items' epilogues
                // (generic-proxy stores, released per warp), before TMA reads them
                if (!__all_sync(0xffffffffu, wait_count(p.h_ready + t.blk, p.h_target, wc))) { ok = false; break; }
                fence_proxy_async_global();
            }
            const CUtensorMap *map_b = &gp_of(t).map_b;
            for (int st = 0; st < n_st; ++st) {
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[slot], ph ^ 1, wc))) { ok = false; break; }
                mbar_arrive_expect_tx_w(&full[slot], b_bytes);
                tma_load_3d_w(b_ring + slot * b_stage, map_b, &full[slot], st * GEMM_KS, t.p0, 0);
                ++issued;
                if (++slot == NS) { slot = 0; ph ^= 1; }
            }
            if constexpr (!SFI) {     // the lo2 pass: boxes from the lo2 plane
                if (ok && item_passes(p, t) > 1) {
                    for (int st = 0; st < n_st; ++st) {
                        if (!__all_sync(0xffffffffu, mbar_wait(&empty[slot], ph ^ 1, wc))) { ok = false; break; }
                        mbar_arrive_expect_tx_w(&full[slot], b_bytes);
                        tma_load_3d_w(b_ring + slot * b_stage, &p.map_b, &full[slot], st * GEMM_KS, t.p0, 2);
                        ++issued;
                        if (++slot == NS) { slot = 0; ph ^= 1; }
                    }
                }
            }
        }
        if (!ok) drain_ring(full, NS, issued, p.wait_limit_ns);
    } else if (warp == 1 || (warp == 2 && n_mma_warps == 2)) {
        // ---------------------------------------------------------------- MMA issue
        // MMA warp m takes the stages st = m, m + n_mma_warps, ... of every
        // work item into its own accumulator; stage g of the CTA (counted
        // over all items) sits in ring slot g % NS with phase parity (g / NS) & 1.
        // A lo2 pass (per-stage mode) issues one MMA per K block over the slot's
        // first plane (lo2) with hi's scale column.
        const int m = warp - 1;
        int db = 0, sb = 0;
        uint32_t dph = 0, sph = 0;
        bool ok = true, issued = false;
        // ring slot and phase parity of the current item's first stage
        int islot = 0;
        uint32_t iph_ring = 0;
        auto advance = [&](int &sl, uint32_t &par, int by) {
            sl += by;
            while (sl >= NS) { sl -= NS; par ^= 1; }
        };
        const bool stacked = SFI || p.stacked;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            Work t;
            item_of(w, t);
            const int n_it = SFI ? n_st : n_st * item_passes(p, t);
            const uint32_t n = stacked ? (uint32_t)(3 * NB) : (uint32_t)t.n_mma;
            // kind::mxf8f6f4 descriptor: A E2M1 (5), B E4M3 (0), both K-major, N >> 3,
            // E8M0 scales, M >> 4; K block kb of a stage takes scale byte kb (fields at 4 and 29)
            const uint32_t idesc0 = (5u << 7) | (0u << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
            uint32_t idesc[4];
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) idesc[kb] = idesc0 | ((uint32_t)kb << 4) | ((uint32_t)kb << 29);
            if (!__all_sync(0xffffffffu, mbar_wait(&d_empty[db], dph ^ 1, wc))) { ok = false; break; }
            if (SFI && !__all_sync(0xffffffffu, mbar_wait(&f_full[sb], sph, wc))) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem + (uint32_t)((m * n_dbuf + db) * d_cols);
            const uint32_t sf_item = tmem + sf_col0 + (uint32_t)(sb * sfi_cols);
            uint32_t acc = 0;
            int slot = islot;
            uint32_t ph = iph_ring;
            advance(slot, ph, m);
            for (int st = m; st < n_st; st += n_mma_warps) {
                if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], ph, wc))) { ok = false; break; }
                tc_fence_after();
                // descriptors of the slot's A and B; K block kb starts 32 bytes further
                // (+2 in the descriptor's address field, which never carries here)
                const uint64_t ad = smem_desc_sw128(smem_addr(a_ring + slot * GEMM_A_STAGE));
                const uint64_t bd = smem_desc_sw128(smem_addr(b_ring + slot * b_stage));
                const uint64_t bd_lo = bd + (uint64_t)(NB * 128 >> 4);
                const uint32_t sf = SFI ? sf_item + (uint32_t)(GEMM_SFI_COLS * st)
                                        : tmem + sf_col0 + (uint32_t)(slot * GEMM_SF_COLS);
                const uint32_t sfb = SFI ? sf + 4 : sf + 8;
                if (st < n_main) {
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        mma_mx_w(d_tmem, ad + 2 * kb, bd + 2 * kb, idesc[kb], sf, sfb, (acc | kb) ? 1u : 0u);
                        if (!stacked) mma_mx_w(d_tmem, ad + 2 * kb, bd_lo + 2 * kb, idesc[kb], sf, sf + 16, 1u);
                    }
                } else {
                    const int nkb = (p.K - n_main * GEMM_KS) / 32;    // the K tail: 1..3 blocks
#pragma unroll
                    for (int kb = 0; kb < 3; ++kb) {
                        if (kb >= nkb) break;
                        mma_mx_w(d_tmem, ad + 2 * kb, bd + 2 * kb, idesc[kb], sf, sfb, (acc | kb) ? 1u : 0u);
                        if (!stacked) mma_mx_w(d_tmem, ad + 2 * kb, bd_lo + 2 * kb, idesc[kb], sf, sf + 16, 1u);
                    }
                }
                acc = 1;
                issued = true;
                mma_commit_w(&empty[slot]);
                advance(slot, ph, n_mma_warps);
            }
            if constexpr (!SFI) {
                // the lo2 pass (one MMA warp): per K block one MMA over the slot's first plane,
                // the lo2 rows, with hi's scale column, into the same accumulator
                if (ok && n_it > n_st) {
                    for (int st = 0; st < n_st; ++st) {
                        if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], ph, wc))) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t ad = smem_desc_sw128(smem_addr(a_ring + slot * GEMM_A_STAGE));
                        const uint64_t bd = smem_desc_sw128(smem_addr(b_ring + slot * b_stage));
                        const uint32_t sf = tmem + sf_col0 + (uint32_t)(slot * GEMM_SF_COLS);
                        const int nkb = st < n_main ? 4 : (p.K - n_main * GEMM_KS) / 32;
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb)
                            if (kb < nkb) mma_mx_w(d_tmem, ad + 2 * kb, bd + 2 * kb, idesc[kb], sf, sf + 8, 1u);
                        mma_commit_w(&empty[slot]);
                        advance(slot, ph, 1);
                    }
                }
            }
            if (!ok) break;
            advance(islot, iph_ring, n_it);
            mma_commit_w(&d_full[m * 2 + db]);
            if (SFI) mma_commit_w(&f_empty[sb]);
            if (++db == n_dbuf) { db = 0; dph ^= 1; }
            if (++sb == 2) { sb = 0; sph ^= 1; }
        }
        if (!ok && issued) {
            mma_commit_w(&drain_bar[m]);
            mbar_wait_drain(&drain_bar[m], 0, p.wait_limit_ns);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------ scale-factor warps
        // Warp q writes TMEM lane quarter q.  A stage's scale factors take 4-column
        // groups: column c of the A group holds, in lane 32q + i, the four E8M0
        // bytes (32-blocks 4st..4st+3) of weight row 32c + i; column c of the B
        // group holds token row 32c + i (stacked: rows of [hi | lo | lo2], lo2 rows
        // taking hi's words).  Per-item mode writes every stage of a work item into
        // an item region once; per-stage mode writes each stage into the slot of its
        // ring stage (both passes of a lo2 item carry the same words: A's, hi's at
        // +8 and lo's at +16).
        const int q = warp & 3;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        int slot = 0, sb = 0;
        uint32_t ph = 0, sph = 0;
        bool ok = true;
        const int n_sfb = p.stacked ? (3 * NB + 31) / 32 : (NB + 31) / 32;
        uint32_t bph = 0;                    // phase parity of the staging barriers (one phase per item)
        // B scale words of K stage kst of item t into v: stacked, word c is row 32c + lane of
        // [hi rows | lo rows | lo2 rows]; otherwise words c and 6 + c are the hi and lo words
        // of token row 32c + lane.  Rows past the block's tokens get 2^0.
        auto load_bsf = [&](const Work &t, int kst, uint32_t (&v)[SF_WORDS]) {
                const uint32_t *bsf = p.b_sf + (size_t)kst * 2 * p.P_max + t.p0;
#pragma unroll
                for (int i = 0; i < SF_WORDS; ++i) v[i] = 0x7F7F7F7Fu;
                if (p.stacked) {
#pragma unroll
                    for (int c = 0; c < SF_WORDS / 2; ++c) {
                        const int r = 32 * c + lane;
                        const int plane = r / NB;
                        const int j = r - plane * NB;
                        if (c < n_sfb && r < 3 * NB && j < t.n_valid)
                            v[c] = __ldg(bsf + (plane == 1 ? (size_t)p.P_max : 0) + j);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < SF_WORDS / 2; ++c) {
                        const int j = 32 * c + lane;
                        if (c < n_sfb && j < t.n_valid) {
                            v[c] = __ldg(bsf + j);
                            v[SF_WORDS / 2 + c] = __ldg(bsf + p.P_max + j);
                        }
                    }
                }
        };
        // per-stage mode: stage st's B words sit in bw[st % SF_PD], loaded SF_PD stages
        // ahead; the slots an item's last stages free take the next item's first stages
        // (a lo2 pass loads its words as it goes)
        uint32_t bw[SF_PD][SF_WORDS];
        if constexpr (!SFI) {
            if constexpr (MODE == MODE_DOWN) pdl_wait();     // h's scales come from the gate/up GEMM
            if (blockIdx.x < total) {
                Work t0;
                item_of(blockIdx.x, t0);
#pragma unroll
                for (int i = 0; i < SF_PD; ++i)
                    if (i < n_st) load_bsf(t0, i, bw[i]);
            }
        }
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            Work t;
            item_of(w, t);
            const int npass = item_passes(p, t);
            if constexpr (!SFI) {
                if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], sph, wc))) { ok = false; break; }
            }
            const uint8_t *sbase = scale_buf + (SFI ? 0 : sb * scale_bytes);
            const uint8_t *srow[4];
            bool row_ok[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                srow[c] = sbase + tile_scale_row(t.up, 32 * c + lane) * KB32;
                row_ok[c] = t.up || t.mb * GEMM_BM + 32 * c + lane < gp_of(t).R;
            }
            // A words of K stage kst: column c
            auto a_words = [&](int kst, uint32_t *v) {
                const int nblk = KB32 - 4 * kst;     // 32-blocks of this stage inside K: 2 or >= 4
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t wv = 0x7F7F7F7Fu;
                    if (row_ok[c]) {
                        const uint16_t *s16 = reinterpret_cast<const uint16_t *>(srow[c] + 4 * kst);
                        const uint32_t lo = s16[0];
                        const uint32_t hi = nblk > 2 ? (uint32_t)s16[1] : 0x7F7Fu;
                        wv = lo | (hi << 16);
                    }
                    v[c] = wv;
                }
            };
            if constexpr (SFI) {
                // The whole item.  The four warps load its A scale bytes (one or two
                // contiguous runs of 16-byte words, a quarter each) and its B scale
                // words (warp q: stages q, q+4, ...), all loads in flight at once, and
                // stage them in shared memory for each other; then each warp writes one
                // 8-column group (A, B) per stage of its lane quarter and waits once.
                const int sf_tid = 32 * q + lane;
                const GemmParams &gq = gp_of(t);
                const int run_bytes = t.up ? 64 * KB32 : min(GEMM_BM, gq.R - t.mb * GEMM_BM) * KB32;
                const int n16 = run_bytes / 16;
                const int n_words = t.up ? 2 * n16 : n16;
                const uint4 *run0 = reinterpret_cast<const uint4 *>(
                    gq.scales + ((size_t)t.e * gq.R + (t.up ? t.mb * 64 : t.mb * GEMM_BM)) * KB32);
                const uint4 *run1 = reinterpret_cast<const uint4 *>(gq.scales + ((size_t)t.e * gq.R + p.F + t.mb * 64) * KB32);
                constexpr int SW = (GEMM_SFI_STAGES_MAX * 4 * GEMM_BM / 16 + 127) / 128;   // words per thread, at most
                uint4 sreg[SW];
#pragma unroll
                for (int i = 0; i < SW; ++i) {
                    const int wi = sf_tid + 128 * i;
                    sreg[i] = make_uint4(0, 0, 0, 0);
                    if (wi < n16) sreg[i] = __ldg(run0 + wi);
                    else if (t.up && wi < n_words) sreg[i] = __ldg(run1 + (wi - n16));
                }
                if constexpr (MODE == MODE_DOWN) pdl_wait();   // h's scales come from the gate/up GEMM
                if (MODE == MODE_FFN && !t.up) {
                    // h's scale words come from this launch's gate/up items of the token block
                    if (!__all_sync(0xffffffffu, wait_count(p.h_ready + t.blk, p.h_target, wc))) { ok = false; break; }
                }
                uint32_t bwr[GEMM_SFI_STAGES_MAX / 4][4];
#pragma unroll
                for (int i = 0; i < GEMM_SFI_STAGES_MAX / 4; ++i) {
                    const int st = q + 4 * i;
                    // stacked block: B column c is row 32c + lane of [hi rows | lo rows | lo2 rows]
                    const uint32_t *bsf = gq.b_sf + (size_t)min(st, n_st - 1) * 2 * p.P_max + t.p0;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int r = 32 * c + lane;
                        const int plane = r / NB;
                        const int j = r - plane * NB;
                        // (in MODE_FFN h's words were written during this launch: a coherent load)
                        const uint32_t *src = bsf + (plane == 1 ? (size_t)p.P_max : 0) + j;
                        bwr[i][c] = st < n_st && c < n_sfb && r < 3 * NB && j < t.n_valid
                                        ? (MODE == MODE_FFN ? __ldcg(src) : __ldg(src)) : 0x7F7F7F7Fu;
                    }
                }
                // the staging buffer is free once all four warps have read the last item's words
                if (!__all_sync(0xffffffffu, mbar_wait(bw_empty, bph ^ 1, wc))) { ok = false; break; }
#pragma unroll
                for (int i = 0; i < GEMM_SFI_STAGES_MAX / 4; ++i) {
                    const int st = q + 4 * i;
                    if (st < n_st) {
#pragma unroll
                        for (int c = 0; c < 4; ++c) bw_s[(st * 4 + c) * 32 + lane] = bwr[i][c];
                    }
                }
#pragma unroll
                for (int i = 0; i < SW; ++i) {
                    const int wi = sf_tid + 128 * i;
                    if (wi < n_words) reinterpret_cast<uint4 *>(scale_buf)[wi] = sreg[i];
                }
                __syncwarp();
                mbar_arrive_w(bw_full);
                if (!__all_sync(0xffffffffu, mbar_wait(f_empty + sb, sph ^ 1, wc))) { ok = false; break; }
                if (!__all_sync(0xffffffffu, mbar_wait(bw_full, bph, wc))) { ok = false; break; }
                tc_fence_after();
                const uint32_t region = lane_base + sf_col0 + (uint32_t)(sb * sfi_cols);
                for (int st = 0; st < n_st; ++st) {
                    uint32_t v[8];
                    a_words(st, v);
#pragma unroll
                    for (int c = 0; c < 4; ++c) v[4 + c] = bw_s[(st * 4 + c) * 32 + lane];
                    tmem_st8(region + (uint32_t)(GEMM_SFI_COLS * st), v);
                }
                __syncwarp();
                mbar_arrive_w(bw_empty);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                mbar_arrive_w(&f_full[sb]);
                bph ^= 1;
            } else {
                Work tn;
                const bool has_next = w + (int)gridDim.x < total;
                if (has_next) item_of(w + gridDim.x, tn);
                for (int st0 = 0; st0 < n_st && ok; st0 += SF_PD) {
#pragma unroll
                    for (int i = 0; i < SF_PD; ++i) {
                        const int st = st0 + i;
                        if (st >= n_st) break;
                        if (!__all_sync(0xffffffffu, mbar_wait(&empty[slot], ph ^ 1, wc))) { ok = false; break; }
                        const uint32_t sf = lane_base + sf_col0 + (uint32_t)(slot * GEMM_SF_COLS);
                        {
                            uint32_t v[4];
                            a_words(st, v);
                            tmem_st4(sf, v);
                        }
                        // B: the hi (and lo) columns of the token block, one store per
                        // 4- or 8-column group (columns past the block's hold 2^0)
                        // (hi words in bw[i][0..5], lo words in bw[i][6..11]; columns 14 and
                        // 15 take two lo words, past any block's hi columns)
                        const uint32_t *b = bw[i];
                        if (p.stacked) {
                            if (n_sfb <= 4) tmem_st4v(sf + 8, b[0], b[1], b[2], b[3]);
                            else tmem_st8v(sf + 8, b[0], b[1], b[2], b[3], b[4], b[5], b[6], b[7]);
                        } else {
                            tmem_st8v(sf + 8, b[0], b[1], b[2], b[3], b[4], b[5], b[6], b[7]);
                            tmem_st4v(sf + 16, b[6], b[7], b[8], b[9]);
                            tmem_st2v(sf + 20, b[10], b[11]);
                        }
                        tmem_wait_st();
                        if (st + SF_PD < n_st) load_bsf(t, st + SF_PD, bw[i]);
                        else if (has_next && i < n_st) load_bsf(tn, i, bw[i]);
                        tc_fence_before();
                        __syncwarp();
                        mbar_arrive_w(&full[slot]);
                        if (++slot == NS) { slot = 0; ph ^= 1; }
                    }
                }
                // the lo2 pass: each stage's A words and hi words again (the lo2 MMAs read
                // hi's scale column), loaded as it goes
                if (ok && npass > 1) {
                    for (int st = 0; st < n_st; ++st) {
                        uint32_t hw[SF_WORDS / 2];
                        const uint32_t *bsf = p.b_sf + (size_t)st * 2 * p.P_max + t.p0;
#pragma unroll
                        for (int c = 0; c < SF_WORDS / 2; ++c) {
                            const int j = 32 * c + lane;
                            hw[c] = c < n_sfb && j < t.n_valid ? __ldg(bsf + j) : 0x7F7F7F7Fu;
                        }
                        if (!__all_sync(0xffffffffu, mbar_wait(&empty[slot], ph ^ 1, wc))) { ok = false; break; }
                        const uint32_t sf = lane_base + sf_col0 + (uint32_t)(slot * GEMM_SF_COLS);
                        uint32_t v[4];
                        a_words(st, v);
                        tmem_st4(sf, v);
                        tmem_st8v(sf + 8, hw[0], hw[1], hw[2], hw[3], hw[4], hw[5], 0x7F7F7F7Fu, 0x7F7F7F7Fu);
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        mbar_arrive_w(&full[slot]);
                        if (++slot == NS) { slot = 0; ph ^= 1; }
                    }
                }
            }
            if (!ok) break;
            if constexpr (!SFI) {
                __syncwarp();
                mbar_arrive_w(&s_empty[sb]);
            }
            if (++sb == 2) { sb = 0; sph ^= 1; }
        }
    } else if (warp >= 8) {
        // ---------------------------------------------------------------- epilogue
        // Two groups of four warps; group eg takes the 16-column chunks
        // eg, eg+2, eg+4, ... of the accumulator.
        const int q = warp & 3;
        const int eg = (warp - 8) >> 2;
        const int tl = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        float *mval = meta_val + (warp - 8) * NB;
        int db = 0;
        uint32_t dph = 0;
        bool ok = true;
        int chunk_par = 0;
        uint32_t ex_ph = 0;                  // bit i: phase parity of exchange buffer i
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            Work t;
            item_of(w, t);
            const GemmParams &gq = gp_of(t);
            const int wrow = tile_weight_row(t.up, tl, t.mb, p.F);
            const bool row_valid = wrow < gq.R;
            // (up) h's lo2 plane: always for stacked blocks, else only where the down GEMM may read it
            bool want_lo2 = t.up && p.stacked;
            if (t.up && !p.stacked && p.down_pass) {
                // the expert's row of the down pass table, one byte per lane (two loads)
                const uint8_t *dp = p.down_pass + (size_t)t.e * DOWN_PASS_STRIDE;
                const bool two = (lane < p.MB_down && __ldg(dp + lane) > 1) ||
                                 (lane + 32 < p.MB_down && __ldg(dp + lane + 32) > 1);
                want_lo2 = __any_sync(0xffffffffu, two);
            }
            const float bias = row_valid ? bf16_to_f32(gq.bias[(size_t)t.e * gq.R + wrow]) : 0.f;
            if (!t.up) {
                for (int c = lane; c < t.n_valid; c += 32) mval[c] = p.row_w[t.p0 + c];
                __syncwarp();
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&d_full[db], dph, wc))) break;
            if (n_mma_warps == 2 && !__all_sync(0xffffffffu, mbar_wait(&d_full[2 + db], dph, wc))) break;
            tc_fence_after();
            // Per-item mode (one accumulator per MMA warp): the accumulator goes back to the
            // MMA warps as soon as this warp has read its last chunk of it, before the
            // chunk's SwiGLU / stores, so the next item's MMAs wait only for the TMEM reads.
            // With two buffers the release comes after the stores (measured faster there).
            bool released = false;
            auto release = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&d_empty[db]);
                released = true;
            };
            if (SFI && 16 * eg >= t.n_mma) release();
            for (int c0 = 16 * eg; c0 < t.n_mma; c0 += 32) {
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = 0.f;
                // the sum over the MMA warps' accumulators and, stacked, their hi, lo and lo2 thirds
                for (int mw = 0; mw < n_mma_warps; ++mw) {
                    const uint32_t d_tmem = lane_base + (uint32_t)((mw * n_dbuf + db) * d_cols);
                    for (int half = 0; half < (p.stacked ? 3 : 1); ++half) {
                        uint32_t v[16];
                        tmem_ld16(d_tmem + (uint32_t)(half * NB + c0), v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc[i] += __uint_as_float(v[i]);
                    }
                }
                if (SFI && c0 + 32 >= t.n_mma) release();
                if (t.up) {
                    // SwiGLU: lanes < 16 hold gate rows, lanes >= 16 the linear rows of the
                    // same h rows; lanes < 16 finish columns 0..7, lanes >= 16 columns 8..15
                    const int half = lane >> 4;
                    float hv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float send = lane < 16 ? acc[8 + i] + bias : acc[i] + bias;
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                        const float gate = lane < 16 ? acc[i] + bias : recv;
                        const float lin = lane < 16 ? recv : acc[8 + i] + bias;
                        const float g = fminf(gate, 7.0f);
                        const float u = fminf(fmaxf(lin, -7.0f), 7.0f);
                        hv[i] = __fdividef(g, 1.0f + __expf(-1.702f * g)) * (u + 1.0f);
                    }
                    // block maxima over the 32 h rows of warps q and q^1 (one 32-block of F)
                    float m[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float a = fabsf(hv[i]);
                        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
                        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
                        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
                        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 8));
                        m[i] = a;
                    }
                    float *ex = amax_s + (eg * 2 + chunk_par) * 4 * 16;     // [4 warps][16 columns]
                    if ((lane & 15) < 8) {
                        float mine = m[0];
#pragma unroll
                        for (int i = 1; i < 8; ++i)
                            if ((lane & 7) == i) mine = m[i];
                        ex[q * 16 + half * 8 + (lane & 7)] = mine;
                    }
                    // all four warps of the group have written their maxima (bounded wait)
                    __syncwarp();
                    mbar_arrive_w(&ex_bar[eg * 2 + chunk_par]);
                    if (!__all_sync(0xffffffffu, mbar_wait(&ex_bar[eg * 2 + chunk_par], (ex_ph >> chunk_par) & 1u, wc))) {
                        ok = false;
                        break;
                    }
                    ex_ph ^= 1u << chunk_par;
#pragma unroll
                    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], ex[(q ^ 1) * 16 + half * 8 + i]);
                    chunk_par ^= 1;
                    const int j = t.mb * 64 + 16 * q + (lane & 15);     // h row (F index)
                    const int fblk = j >> 5;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int col = c0 + half * 8 + i;
                        const int s_hi = e4m3_block_exp(m[i]);
                        const int s_lo = max(s_hi - 4, -126);
                        const float v = hv[i];
                        // the three terms; each residual is exact in fp32
                        const uint32_t qh = f32x2_to_e4m3x2(v * pow2f(-s_hi), 0.0f) & 0xFFu;
                        const float res = v - e4m3_to_f32(qh) * pow2f(s_hi);
                        const uint32_t ql = f32x2_to_e4m3x2(res * pow2f(-s_lo), 0.0f) & 0xFFu;
                        if (col < t.n_valid) {
                            const size_t prow = (size_t)(t.p0 + col);
                            p.h_q[prow * p.Kf + j] = (uint8_t)qh;
                            p.h_q[((size_t)p.P_max + prow) * p.Kf + j] = (uint8_t)ql;
                            if (want_lo2) {
                                const float res2 = res - e4m3_to_f32(ql) * pow2f(s_lo);
                                const uint32_t ql2 = f32x2_to_e4m3x2(res2 * pow2f(-s_hi), 0.0f) & 0xFFu;
                                p.h_q[((size_t)2 * p.P_max + prow) * p.Kf + j] = (uint8_t)ql2;
                            }
                            if ((q & 1) == 0 && (lane & 15) == 0) {
                                // one lane per (column, 32-block): the two scale bytes
                                const size_t wi = (size_t)(fblk >> 2) * 2 * p.P_max;
                                p.h_sf[(wi + prow) * 4 + (fblk & 3)] = (uint8_t)(s_hi + 127);
                                p.h_sf[(wi + p.P_max + prow) * 4 + (fblk & 3)] = (uint8_t)(s_lo + 127);
                            }
                        }
                    }
                } else {
                    // weighted expert output w * (W2 h + b2), one expert-sorted row per column
                    if (row_valid) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < t.n_valid)
                                gq.out_rows[(size_t)(t.p0 + c0 + i) * gq.R + wrow] = (acc[i] + bias) * mval[c0 + i];
                    }
                }
            }
            if (!ok) break;
            if (MODE == MODE_FFN && t.up) {
                // this warp's h rows of the token block are written: release them to the down
                // items (each lane's stores fenced, then one count per warp)
                fence_proxy_async_global();
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(p.h_ready + t.blk, 1u);
            }
            if (!released) release();
            if (++db == n_dbuf) { db = 0; dph ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template __global__ void expert_gemm_kernel<MODE_UP, false>(const __grid_constant__ GemmParams p,
                                                              const __grid_constant__ GemmParams p2);
template __global__ void expert_gemm_kernel<MODE_UP, true>(const __grid_constant__ GemmParams p,
                                                             const __grid_constant__ GemmParams p2);
template __global__ void expert_gemm_kernel<MODE_DOWN, false>(const __grid_constant__ GemmParams p,
                                                                const __grid_constant__ GemmParams p2);
template __global__ void expert_gemm_kernel<MODE_DOWN, true>(const __grid_constant__ GemmParams p,
                                                               const __grid_constant__ GemmParams p2);
template __global__ void expert_gemm_kernel<MODE_FFN, true>(const __grid_constant__ GemmParams p,
                                                              const __grid_constant__ GemmParams p2);

// The pass table of the large-block GEMMs: for every gate/up work-item weight
// block (64 gate rows and their 64 linear rows of W13) and every down weight
// block (128 rows of W2), 2 when a scale byte of its rows reaches LO2_SCALE_MIN
// (a pass over the lo2 term), else 1.  One warp per block, all of a lane's
// loads in flight together.  It reads weights only, so it runs at once; it
// waits for the kernel before it only at its end, which keeps the stream's
// order for the GEMM after it.
__global__ void __launch_bounds__(256) pass_plan_kernel(const uint8_t *w13_scales, const uint8_t *w2_scales, int E,
                                                        int d, int F, uint8_t *up_pass, uint8_t *down_pass) {
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int mb_up = F / 64, mb_dn = (d + GEMM_BM - 1) / GEMM_BM;
    const long long n_up = (long long)E * mb_up, n_dn = (long long)E * mb_dn;
    if (gw < n_up + n_dn) {
        const uint4 *run[2];
        int n16[2];
        if (gw < n_up) {
            const int e = (int)(gw / mb_up), mb = (int)(gw % mb_up);
            const size_t kb = (size_t)d / 32;
            run[0] = reinterpret_cast<const uint4 *>(w13_scales + ((size_t)e * 2 * F + (size_t)mb * 64) * kb);
            run[1] = reinterpret_cast<const uint4 *>(w13_scales + ((size_t)e * 2 * F + F + (size_t)mb * 64) * kb);
            n16[0] = n16[1] = (int)(64 * kb / 16);
        } else {
            const long long g = gw - n_up;
            const int e = (int)(g / mb_dn), mb = (int)(g % mb_dn);
            const size_t kb = (size_t)F / 32;
            const int rows = min(GEMM_BM, d - mb * GEMM_BM);
            run[0] = reinterpret_cast<const uint4 *>(w2_scales + ((size_t)e * d + (size_t)mb * GEMM_BM) * kb);
            run[1] = run[0];
            n16[0] = (int)(rows * kb / 16);
            n16[1] = 0;
        }
        uint32_t m4 = 0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            for (int i0 = lane; i0 < n16[r]; i0 += 32 * 8) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + 32 * u;
                    v[u] = i < n16[r] ? __ldg(run[r] + i) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) m4 = __vmaxu4(m4, __vmaxu4(__vmaxu4(v[u].x, v[u].y), __vmaxu4(v[u].z, v[u].w)));
            }
        }
        uint32_t m = max(max(m4 & 0xFFu, (m4 >> 8) & 0xFFu), max((m4 >> 16) & 0xFFu, m4 >> 24));
        m = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) {
            const uint8_t np = m >= (uint32_t)LO2_SCALE_MIN ? 2 : 1;
            if (gw < n_up) {
                up_pass[gw] = np;
            } else {
                const long long g = gw - n_up;
                down_pass[(g / mb_dn) * DOWN_PASS_STRIDE + g % mb_dn] = np;
            }
        }
    }
    pdl_wait();
}

cudaError_t launch_pass_plan(const uint8_t *w13_scales, const uint8_t *w2_scales, int E, int d, int F,
                             uint8_t *up_pass, uint8_t *down_pass, cudaStream_t s) {
    const long long warps = (long long)E * (F / 64) + (long long)E * ((d + GEMM_BM - 1) / GEMM_BM);
    return launch_pdl(pass_plan_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, w13_scales, w2_scales, E,
                      d, F, up_pass, down_pass);
}

template <int MODE, bool SFI>
static cudaError_t launch_gemm_t(const GemmParams &p, const GemmParams &p2, int grid, int smem, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<MODE, SFI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(expert_gemm_kernel<MODE, SFI>, dim3(grid), dim3(GEMM_THREADS), (size_t)smem, s, p, p2);
}

cudaError_t launch_expert_gemm(int mode, const GemmParams &p, int grid, int smem, cudaStream_t s) {
    if (mode == MODE_UP)
        return p.sf_item ? launch_gemm_t<MODE_UP, true>(p, p, grid, smem, s)
                         : launch_gemm_t<MODE_UP, false>(p, p, grid, smem, s);
    return p.sf_item ? launch_gemm_t<MODE_DOWN, true>(p, p, grid, smem, s)
                     : launch_gemm_t<MODE_DOWN, false>(p, p, grid, smem, s);
}

// Both GEMMs of a decode-sized batch in one launch (per-item scale factors, d_model == d_ff):
// pu the gate/up GEMM with h_ready / h_target set, pd the down GEMM.
cudaError_t launch_expert_ffn(const GemmParams &pu, const GemmParams &pd, int grid, int smem, cudaStream_t s) {
    if (!pu.sf_item || !pd.sf_item || pu.K != pd.K || !pu.h_ready) return cudaErrorInvalidValue;
    return launch_gemm_t<MODE_FFN, true>(pu, pd, grid, smem, s);
}

}  // namespace moe
