// Grouped MXFP4-weight GEMMs of the MoE experts on sm_100a (tcgen05 + TMEM + TMA).
//
// One persistent CTA per SM walks the work items (expert e, 128-row weight
// block, block of up to 256 tokens routed to e).  For each item:
//   A (weights, M = 128 rows): packed E2M1 codes arrive by TMA (128-byte
//     swizzle) into a shared-memory ring; the E8M0 scales of the 128 rows by
//     one untiled bulk copy.  Decoder warps convert 64 K-elements per row at a
//     time to fp16 (hardware e2m1x2 conversion times the block's power of
//     two, relative to a per-row power of two that keeps every block of the
//     row exact in fp16) and store them straight into tensor memory, where
//     the MMA reads A ("A from TMEM" form).  The decoded weights never touch
//     shared memory, so shared-memory bandwidth is left to the codes and B.
//   B (activations, N = tokens, K-major fp16): TMA boxes of up to 64
//     expert-sorted rows (the sorted copy of the normalised tokens for the
//     gate/up GEMM, h for the down GEMM) into a shared-memory ring in the
//     128-byte swizzled canonical layout.
//   D (fp32, 128 lanes x N columns) accumulates in TMEM.  A tcgen05.mma
//     occupies its issuing thread for about 120 cycles whatever N is, so small
//     token blocks are spread over up to three MMA warps, each accumulating
//     every third sub-stage into its own accumulator; the epilogue sums them.
// Gate/up epilogue: z = D * 2^c * rho_token + b13, clamped SwiGLU
//   h = min(g,7) * sigmoid(1.702 min(g,7)) * (clamp(u,-7,7) + 1)
//   ("gpt-oss-20B" hub page, section 3.3); each 128-row block holds 64 gate
//   rows and their 64 linear rows so the pair meets in one warp.
// Down epilogue: o = w_token * (D * 2^c + b2) written to the pair's
//   expert-sorted row; the combine kernel adds a token's rows to its residual
//   (weighted combine, "gpt-oss-20B" page section 3.4; pnsm.cn overview 2.2).
//
// Warp roles (672 threads): 0 codes/scales producer, 20 B producer (TMA
// instructions hold their issuing thread too, so the two streams get their
// own threads), 1-3 MMA issue (3 also allocates TMEM), 4-7 and 12-15
// decoder groups, 8-11 epilogue group; warps 16-19 are a third decoder group
// for small token blocks (several MMA warps) and a second epilogue group
// otherwise.  Decoder groups take two-sub-stage chunks in turn; epilogue
// groups take 16-column chunks in turn.  The decoders hand each row's power-of-two shift to the
// epilogue through shared memory.  Every mbarrier wait is bounded (WaitCtl);
// when one runs out the CTA stops issuing work, drains its copies and MMAs in
// flight, frees TMEM and returns with the error latched.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

struct Work {
    int e, mb, p0, n_valid, n_mma;
};

__device__ __forceinline__ void work_of(int w, const int *tiles_s, const int *counts_s, const int *offsets_s, int E,
                                        int MB, int nb_rows, Work &t) {
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
    t.p0 = offsets_s[e] + nb * nb_rows;
    t.n_valid = min(nb_rows, counts_s[e] - nb * nb_rows);
    t.n_mma = (t.n_valid + 15) & ~15;
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

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Largest and smallest E8M0 byte of a row (255 excluded from the largest; a
// 255 makes the smallest -1), n even, row 2-byte aligned.
__device__ __forceinline__ void row_scale_range(const uint8_t *s, int n, int &mx, int &mn) {
    const uint16_t *w = reinterpret_cast<const uint16_t *>(s);
    mx = -1;
    mn = 256;
#pragma unroll 8
    for (int b = 0; b < n / 2; ++b) {
        const uint32_t v = w[b];
        const int lo = (int)(v & 0xFFu), hi = (int)(v >> 8);
        mx = max(mx, lo == 255 ? -1 : lo);
        mx = max(mx, hi == 255 ? -1 : hi);
        mn = min(mn, lo == 255 ? -1 : lo);
        mn = min(mn, hi == 255 ? -1 : hi);
    }
}

// Largest E8M0 byte (other than 255) of a row's n scale bytes (n even, row
// 2-byte aligned), read as 16-bit words so the loads pipeline.
__device__ __forceinline__ int row_scale_max(const uint8_t *s, int n) {
    const uint16_t *w = reinterpret_cast<const uint16_t *>(s);
    int m = -1;
#pragma unroll 8
    for (int b = 0; b < n / 2; ++b) {
        const uint32_t v = w[b];
        const int lo = (int)(v & 0xFFu), hi = (int)(v >> 8);
        m = max(m, lo == 255 ? -1 : lo);
        m = max(m, hi == 255 ? -1 : hi);
    }
    return m;
}

template <int MODE>
__global__ void __launch_bounds__(GEMM_THREADS, 1) expert_gemm_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int U = p.b_unit;
    const int b_slot_bytes = U * p.b_stage_bytes;
    const GemmSmem plan = gemm_smem_plan(p.K, p.E, p.n_c_stages, p.n_a_slots, p.n_b_stages, b_slot_bytes);
    const int SC = p.n_c_stages, NA = p.n_a_slots, NBS = p.n_b_stages, NI = p.n_iss;
    const int NP = NA / 2;                 // A slot pairs: one pair per decoder chunk of two sub-stages
    const int NG = p.n_dec_groups;         // decoder groups
    const int NEG = NG == 3 ? 1 : 2;       // epilogue groups
    const int PPG = NP / NG;               // slot pairs owned by each decoder group
    // Chunk gc (two sub-stages of a code stage) is decoded by group gc % NG into
    // the group's pair (gc / NG) % PPG and its MMAs are issued by MMA warp
    // (gc % NG) % NI, so each decoder group and its MMA warp form one pipeline.
    uint8_t *code_ring = smem + plan.code_off;
    uint8_t *b_ring = smem + plan.b_off;
    uint8_t *scale_buf = smem + plan.scale_off;
    const int scale_bytes = align_up(GEMM_BM * (p.K / 32), 128);
    float *meta_val = reinterpret_cast<float *>(smem + plan.meta_off);    // [8 warps][NB_MAX / 2]
    int *tok_s = reinterpret_cast<int *>(smem + plan.tok_off);            // [NB_MAX]
    int *shift_s = reinterpret_cast<int *>(smem + plan.shift_off);        // [2][128]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + plan.bar_off);
    uint64_t *c_full = bars;
    uint64_t *c_empty = c_full + SC;
    uint64_t *s_full = c_empty + SC;
    uint64_t *s_empty = s_full + 2;
    uint64_t *a_full = s_empty + 2;
    uint64_t *a_empty = a_full + NA;
    uint64_t *b_full = a_empty + NA;
    uint64_t *b_empty = b_full + NBS;
    uint64_t *d_full = b_empty + NBS;
    uint64_t *d_empty = d_full + 2;
    uint64_t *h_full = d_empty + 2;
    uint64_t *h_empty = h_full + 2;
    uint64_t *drain_bar = h_empty + 2;                                     // [GEMM_ISS_MAX]
    uint32_t *tmem_base_s = reinterpret_cast<uint32_t *>(smem + plan.misc_off);
    volatile int *abort_s = reinterpret_cast<volatile int *>(smem + plan.misc_off + 4);
    int *counts_s = reinterpret_cast<int *>(smem + plan.misc_off + 16);
    int *offsets_s = counts_s + (p.E + 1);
    int *tiles_s = offsets_s + (p.E + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB32 = p.K / 32;
    const int n_sub = p.K / GEMM_KA;
    const int n_cstages = (p.K + GEMM_KS - 1) / GEMM_KS;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SC; ++i) {
            mbar_init(&c_full[i], 1);
            mbar_init(&c_empty[i], 4 * NG);   // every decoder warp
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 4 * NG);
            mbar_init(&d_full[i], NI);        // one commit per MMA warp
            mbar_init(&d_empty[i], 4 * NEG);  // every epilogue warp
            mbar_init(&h_full[i], 4);
            mbar_init(&h_empty[i], 4 * NEG);
        }
        for (int i = 0; i < NP; ++i) {
            mbar_init(&a_full[i], 4);         // the four warps of the group that decoded the pair
            mbar_init(&a_empty[i], 1);        // the commit of the MMA warp that consumed it
        }
        for (int i = 0; i < NBS; ++i) {
            mbar_init(&b_full[i], 1);
            mbar_init(&b_empty[i], U);     // one commit per sub-stage of the slot
        }
        for (int i = 0; i < GEMM_ISS_MAX; ++i) mbar_init(&drain_bar[i], 1);
        *abort_s = 0;
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
        counts_s[i] = i < p.E ? p.counts[i] : 0;
        offsets_s[i] = p.offsets[i];
        tiles_s[i] = p.tiles[i];
    }
    if (warp == 3) {
        tmem_alloc(tmem_base_s, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_s;
    const int total = p.MB * tiles_s[p.E];
    const WaitCtl wc{abort_s, p.err, MODE == MODE_UP ? (unsigned)ERR_WAIT_UP : (unsigned)ERR_WAIT_DOWN,
                     p.wait_limit_ns};
    // accumulator of MMA warp i in buffer set db: columns NA*32 + (db*NI + i)*nb_rows
    const uint32_t d_col0 = (uint32_t)(NA * 32);

    if (warp == 0) {
        // ------------------------------------------------ codes + scales producer
        if (lane == 0) {
            tma_prefetch_desc(&p.map_codes);
            int cslot = 0, sb = 0;
            uint32_t cph = 0, sph = 0;
            long long c_issued = 0, s_issued = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                Work t;
                work_of(w, tiles_s, counts_s, offsets_s, p.E, p.MB, p.nb_rows, t);
                if (!mbar_wait(&s_empty[sb], sph ^ 1, wc)) { ok = false; break; }
                uint8_t *sdst = scale_buf + sb * scale_bytes;
                if (MODE == MODE_UP) {
                    const int j0 = t.mb * 64;
                    const uint32_t bytes = 64u * KB32;
                    mbar_arrive_expect_tx(&s_full[sb], 2 * bytes);
                    bulk_load(sdst, p.scales + ((size_t)t.e * p.R + j0) * KB32, bytes, &s_full[sb]);
                    bulk_load(sdst + bytes, p.scales + ((size_t)t.e * p.R + p.F + j0) * KB32, bytes, &s_full[sb]);
                } else {
                    const int m0 = t.mb * GEMM_BM;
                    const uint32_t bytes = (uint32_t)min(GEMM_BM, p.R - m0) * KB32;
                    mbar_arrive_expect_tx(&s_full[sb], bytes);
                    bulk_load(sdst, p.scales + ((size_t)t.e * p.R + m0) * KB32, bytes, &s_full[sb]);
                }
                ++s_issued;
                if (++sb == 2) { sb = 0; sph ^= 1; }
                for (int ks = 0; ks < n_cstages; ++ks) {
                    if (!mbar_wait(&c_empty[cslot], cph ^ 1, wc)) { ok = false; break; }
                    uint8_t *cdst = code_ring + cslot * GEMM_CODE_STAGE;
                    mbar_arrive_expect_tx(&c_full[cslot], GEMM_CODE_STAGE);
                    if (MODE == MODE_UP) {
                        tma_load_3d(cdst, &p.map_codes, &c_full[cslot], ks * 128, t.mb * 64, t.e);
                        tma_load_3d(cdst + 64 * 128, &p.map_codes, &c_full[cslot], ks * 128, p.F + t.mb * 64, t.e);
                    } else {
                        tma_load_3d(cdst, &p.map_codes, &c_full[cslot], ks * 128, t.mb * GEMM_BM, t.e);
                    }
                    ++c_issued;
                    if (++cslot == SC) { cslot = 0; cph ^= 1; }
                }
            }
            if (!ok) {
                drain_ring(c_full, SC, c_issued, p.wait_limit_ns);
                drain_ring(s_full, 2, s_issued, p.wait_limit_ns);
            }
        }
    } else if (warp == 20) {
        // ------------------------------------------------------------ B producer
        // One slot holds U consecutive 64-K blocks of the work item's token
        // rows; with U = 4 a single 3-D TMA box fills it.
        if (lane == 0) {
            tma_prefetch_desc(&p.map_b);
            int bslot = 0;
            uint32_t bph = 0;
            long long b_issued = 0;
            bool ok = true;
            const int box = p.b_box_rows;
            const int n_units = (n_sub + U - 1) / U;
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                Work t;
                work_of(w, tiles_s, counts_s, offsets_s, p.E, p.MB, p.nb_rows, t);
                const int nbox = (t.n_mma + box - 1) / box;
                for (int u = 0; u < n_units; ++u) {
                    if (!mbar_wait(&b_empty[bslot], bph ^ 1, wc)) { ok = false; break; }
                    uint8_t *bdst = b_ring + bslot * b_slot_bytes;
                    mbar_arrive_expect_tx(&b_full[bslot], (uint32_t)(nbox * box * 128 * U));
                    for (int g = 0; g < nbox; ++g)
                        tma_load_3d(bdst + g * box * 128 * U, &p.map_b, &b_full[bslot], 0, t.p0 + box * g, u * U);
                    // a slot past the last K block is consumed fewer than U times
                    for (int r = min(U, n_sub - u * U); r < U; ++r) mbar_arrive(&b_empty[bslot]);
                    ++b_issued;
                    if (++bslot == NBS) { bslot = 0; bph ^= 1; }
                }
            }
            if (!ok) drain_ring(b_full, NBS, b_issued, p.wait_limit_ns);
        }
    } else if (warp >= 1 && warp <= 3) {
        // ------------------------------------------- MMA issue: warp i-1 takes sub-stages i-1, i-1+NI, ...
        const int mi = warp - 1;
        if (lane == 0 && mi < NI) {
            int db = 0;
            uint32_t dph = 0;
            // Running counters instead of divisions (a 64-bit division is a long
            // software routine): the decoder group of the next chunk, each
            // group's next pair and its phase, and the next B fill.
            int turn = 0;                          // decoder group of the next chunk
            int pp0 = 0, pp1 = 0, pp2 = 0;         // next pair (within its group) of groups 0..2
            uint32_t ph0 = 0, ph1 = 0, ph2 = 0;    // phase parity of that pair
            int ub = 0, bslot = 0;                 // next B fill (within the work item) and its slot
            uint32_t bph = 0;
            const int ushift = U == 4 ? 2 : 0;
            const int n_units = (n_sub + U - 1) / U;
            const int n_chunks = (n_sub + 1) / 2;  // two per full code stage, ceil(r/2) for a tail of r
            bool ok = true, issued = false;
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                Work t;
                work_of(w, tiles_s, counts_s, offsets_s, p.E, p.MB, p.nb_rows, t);
                const uint32_t idesc = idesc_f16_f32(GEMM_BM, (uint32_t)t.n_mma);
                if (!mbar_wait(&d_empty[db], dph ^ 1, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem + d_col0 + (uint32_t)((db * NI + mi) * p.nb_rows);
                bool first = true;
                int u_base = 0;                    // B fills consumed before this work item, relative
                for (int ci = 0; ci < n_chunks && ok; ++ci) {
                    const int grp = turn;
                    turn = turn + 1 == NG ? 0 : turn + 1;
                    const int lp = grp == 0 ? pp0 : (grp == 1 ? pp1 : pp2);
                    const uint32_t lph = grp == 0 ? ph0 : (grp == 1 ? ph1 : ph2);
                    {
                        int np_ = lp + 1;
                        uint32_t nph = lph;
                        if (np_ == PPG) { np_ = 0; nph ^= 1; }
                        if (grp == 0) { pp0 = np_; ph0 = nph; } else if (grp == 1) { pp1 = np_; ph1 = nph; } else { pp2 = np_; ph2 = nph; }
                    }
                    if (grp % NI != mi) continue;
                    const int pair = grp * PPG + lp;
                    if (!mbar_wait(&a_full[pair], lph, wc)) { ok = false; break; }
                    // sub-stages of chunk ci: 2 per code stage, the tail stage may hold 1..4
                    const int j0 = 4 * (ci >> 1) + 2 * (ci & 1);
                    const int na = min(2, n_sub - j0);
                    for (int u = 0; u < na; ++u) {
                        const int j = j0 + u;
                        const int target = j >> ushift;        // B fill of sub-stage j within the work item
                        while (ub < u_base + target) {
                            ++ub;
                            if (++bslot == NBS) { bslot = 0; bph ^= 1; }
                        }
                        if (!mbar_wait(&b_full[bslot], bph, wc)) { ok = false; break; }
                        tc_fence_after();
                        // sub-stage block j % U of the slot
                        const uint32_t b_addr =
                            smem_addr(b_ring + bslot * b_slot_bytes + (j & (U - 1)) * p.b_stage_bytes);
                        const uint32_t a_tmem = tmem + (uint32_t)((2 * pair + u) * 32);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            mma_f16_ts(d_tmem, a_tmem + kk * 8, smem_desc_sw128(b_addr + kk * 32), idesc,
                                       first ? 0u : 1u);
                            first = false;
                        }
                        issued = true;
                        mma_commit(&b_empty[bslot]);
                    }
                    if (!ok) break;
                    mma_commit(&a_empty[pair]);
                }
                if (!ok) break;
                // move the B counters to the first fill of the next work item
                while (ub < u_base + n_units) {
                    ++ub;
                    if (++bslot == NBS) { bslot = 0; bph ^= 1; }
                }
                ub -= u_base + n_units;
                mma_commit(&d_full[db]);
                if (++db == p.n_d_bufs) { db = 0; dph ^= 1; }
            }
            if (!ok && issued) {
                mma_commit(&drain_bar[mi]);
                mbar_wait_drain(&drain_bar[mi], 0, p.wait_limit_ns);
            }
        }
    } else if ((warp >= 4 && warp < 8) || (warp >= 12 && warp < 16 && NG >= 2) || (warp >= 16 && warp < 20 && NG == 3)) {
        // ------------------------------------------------------------ decoders
        // NG groups of four warps.  Each code stage (4 sub-stages of 64 K
        // elements) is cut into chunks of two sub-stages; chunk gc goes to
        // group gc mod NG and fills one of the group's own A slot pairs (TMEM
        // lanes 32q..32q+31 of its warps), with one handshake per chunk.
        const int q = warp & 3;
        const int grp = warp < 8 ? 0 : (warp < 16 ? 1 : 2);
        const int tl = 32 * q + lane;                           // TMEM lane = A row
        const int my_row = MODE == MODE_UP ? (16 * q + (lane & 15) + (lane >= 16 ? 64 : 0)) : tl;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        int cslot = 0, sb = 0, hb = 0;
        uint32_t cph = 0, sph = 0, hph = 0;
        int turn = 0;                                           // decoder group of the next chunk
        int mpair = 0;                                          // this group's next pair (within the group)
        uint32_t mph = 0;                                       // and its phase parity
        bool ok = true;
        for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
            Work t;
            work_of(w, tiles_s, counts_s, offsets_s, p.E, p.MB, p.nb_rows, t);
            const bool row_valid = MODE == MODE_UP || (t.mb * GEMM_BM + my_row < p.R);
            if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], sph, wc))) { ok = false; break; }
            const uint8_t *srow = scale_buf + sb * scale_bytes + my_row * KB32;
            int smax = -1, smin = 256;
            if (row_valid) row_scale_range(srow, KB32, smax, smin);
            const int c = row_shift_from_max(smax);
            const bool fast = row_valid && smin >= smax - 27;   // every block multiplier is a normal fp16
            if (grp == 0) {
                // hand the row shift to the epilogue
                if (!__all_sync(0xffffffffu, mbar_wait(&h_empty[hb], hph ^ 1, wc))) { ok = false; break; }
                shift_s[hb * GEMM_BM + tl] = c;
                __syncwarp();
                if (lane == 0) mbar_arrive(&h_full[hb]);
                if (++hb == 2) { hb = 0; hph ^= 1; }
            }
            for (int ks = 0; ks < n_cstages && ok; ++ks) {
                if (!__all_sync(0xffffffffu, mbar_wait(&c_full[cslot], cph, wc))) { ok = false; break; }
                const uint8_t *crow = code_ring + cslot * GEMM_CODE_STAGE + my_row * 128;
                const int nsub = min(4, (p.K - ks * GEMM_KS) / GEMM_KA);
                // the 8 block multipliers of this code stage
                uint32_t mult[8];
                {
                    const uint16_t *sw16 = reinterpret_cast<const uint16_t *>(srow + ks * 8);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t v = (2 * i < 2 * nsub) ? (uint32_t)sw16[i] : 0x7F7Fu;
                        const int s0 = (int)(v & 0xFFu), s1 = (int)(v >> 8);
                        if (fast) {
                            mult[2 * i] = block_multiplier_fast(s0, smax);
                            mult[2 * i + 1] = block_multiplier_fast(s1, smax);
                        } else {
                            mult[2 * i] = block_multiplier(s0, c);
                            mult[2 * i + 1] = block_multiplier(s1, c);
                        }
                    }
                }
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int a0 = 2 * cc;
                    if (a0 >= nsub) break;
                    const int na = min(2, nsub - a0);
                    const bool mine = turn == grp;
                    turn = turn + 1 == NG ? 0 : turn + 1;
                    if (!mine) continue;
                    const int pair = grp * PPG + mpair;
                    const uint32_t pph = mph;
                    if (++mpair == PPG) { mpair = 0; mph ^= 1; }
                    if (!__all_sync(0xffffffffu, mbar_wait(&a_empty[pair], pph ^ 1, wc))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int sw = my_row & 7;
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        if (u < na) {
                            const int a = a0 + u;
                            uint32_t out[32];
                            if (row_valid) {
                                const uint4 w0 = *reinterpret_cast<const uint4 *>(crow + (((2 * a) ^ sw) << 4));
                                const uint4 w1 = *reinterpret_cast<const uint4 *>(crow + (((2 * a + 1) ^ sw) << 4));
                                const uint32_t m0 = mult[2 * a], m1 = mult[2 * a + 1];
                                const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    uint32_t h4[4];
                                    e2m1x8_to_half2x4(words[i], h4);
#pragma unroll
                                    for (int jj = 0; jj < 4; ++jj) out[4 * i + jj] = hmul2_u32(h4[jj], i < 4 ? m0 : m1);
                                }
                            } else {
#pragma unroll
                                for (int i = 0; i < 32; ++i) out[i] = 0u;
                            }
                            tmem_st32(lane_base + (uint32_t)((2 * pair + u) * 32), out);
                        }
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&a_full[pair]);
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&c_empty[cslot]);
                if (++cslot == SC) { cslot = 0; cph ^= 1; }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[sb]);
            if (++sb == 2) { sb = 0; sph ^= 1; }
        }
    } else if ((warp >= 8 && warp < 12) || (warp >= 16 && warp < 20 && NG < 3)) {
        // ------------------------------------------------------------- epilogue
        // Two groups of four warps; group eg takes the 16-column chunks
        // eg, eg+2, eg+4, ... of the accumulators, summing the MMA warps' parts.
        const int q = warp & 3;
        const int eg = warp >= 16 ? 1 : 0;
        const int tl = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        float *mval = meta_val + (eg * 4 + q) * (GEMM_NB_MAX / 2);      // value of chunk m's column i at [(m/2)*16 + i]
        int db = 0, hb = 0;
        uint32_t dph = 0, hph = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            Work t;
            work_of(w, tiles_s, counts_s, offsets_s, p.E, p.MB, p.nb_rows, t);
            int row;
            bool row_valid;
            if (MODE == MODE_UP) {
                row = (lane < 16 ? 0 : p.F) + t.mb * 64 + 16 * q + (lane & 15);
                row_valid = true;
            } else {
                row = t.mb * GEMM_BM + tl;
                row_valid = row < p.R;
            }
            const float bias = row_valid ? bf16_to_f32(p.bias[(size_t)t.e * p.R + row]) : 0.f;
            // per-column rho (UP) or routing weight (DOWN) of this group's columns
            for (int cc = lane; cc < GEMM_NB_MAX / 2; cc += 32) {
                const int col = ((cc >> 4) * NEG + eg) * 16 + (cc & 15);
                if (col < t.n_mma) {
                    const int pr = t.p0 + min(col, t.n_valid - 1);
                    mval[cc] = MODE == MODE_UP ? p.rho[p.row_token[pr]] : p.row_w[pr];
                }
            }
            __syncwarp();
            if (!__all_sync(0xffffffffu, mbar_wait(&h_full[hb], hph, wc))) break;
            const float cscale = exp2i(shift_s[hb * GEMM_BM + tl]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&h_empty[hb]);
            if (++hb == 2) { hb = 0; hph ^= 1; }
            if (!__all_sync(0xffffffffu, mbar_wait(&d_full[db], dph, wc))) break;
            tc_fence_after();
            const uint32_t d_tmem = lane_base + d_col0 + (uint32_t)(db * NI * p.nb_rows);
            for (int c0 = 16 * eg; c0 < t.n_mma; c0 += 16 * NEG) {
                float acc[16];
                {
                    uint32_t v[16];
                    tmem_ld16(d_tmem + (uint32_t)c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[i] = __uint_as_float(v[i]);
                }
                for (int mi = 1; mi < NI; ++mi) {
                    uint32_t v[16];
                    tmem_ld16(d_tmem + (uint32_t)(mi * p.nb_rows + c0), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[i] += __uint_as_float(v[i]);
                }
                const float *mv = mval + (c0 / (16 * NEG)) * 16;
                if (MODE == MODE_UP) {
                    float z[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) z[i] = acc[i] * (cscale * mv[i]) + bias;
                    __half *hout = reinterpret_cast<__half *>(p.out);
                    const int jrow = t.mb * 64 + 16 * q + (lane & 15);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float send = lane < 16 ? z[8 + i] : z[i];
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                        const float gate = lane < 16 ? z[i] : recv;
                        const float lin = lane < 16 ? recv : z[8 + i];
                        const int col = c0 + (lane < 16 ? i : 8 + i);
                        const float g = fminf(gate, 7.0f);
                        const float u = fminf(fmaxf(lin, -7.0f), 7.0f);
                        const float h = __fdividef(g, 1.0f + __expf(-1.702f * g)) * (u + 1.0f);
                        if (col < t.n_valid)
                            hout[((size_t)t.mb * p.b_rows_total + t.p0 + col) * 64 + (jrow - t.mb * 64)] =
                                __float2half_rn(h);
                    }
                } else {
                    // weighted expert output w * (W2 h + b2), one expert-sorted row per column
                    float *o = reinterpret_cast<float *>(p.out);
                    if (row_valid) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < t.n_valid)
                                o[(size_t)(t.p0 + c0 + i) * p.out_ld + row] = (acc[i] * cscale + bias) * mv[i];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[db]);
            if (++db == p.n_d_bufs) { db = 0; dph ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template __global__ void expert_gemm_kernel<MODE_UP>(const __grid_constant__ GemmParams p);
template __global__ void expert_gemm_kernel<MODE_DOWN>(const __grid_constant__ GemmParams p);

}  // namespace moe

namespace moe {

cudaError_t launch_expert_gemm(int mode, const GemmParams &p, int grid, int smem, cudaStream_t s) {
    if (mode == MODE_UP) {
        cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<MODE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        expert_gemm_kernel<MODE_UP><<<grid, GEMM_THREADS, smem, s>>>(p);
    } else {
        cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<MODE_DOWN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        expert_gemm_kernel<MODE_DOWN><<<grid, GEMM_THREADS, smem, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace moe
