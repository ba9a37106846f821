// Routing side of the MoE block on sm_100a:
//   route_fma_kernel RMSNorm + router logits + top-k + softmax over the chosen,
//                    plus the fp32 normalised tokens for the experts; eight
//                    tokens per CTA, the router on CUDA cores;
//   route_small_kernel  the same for decode-sized batches, a CTA per (token,
//                    16 experts);
//   group_permute_kernel  expert histogram, exclusive scan and a stable
//                    permutation of the (token, expert) pairs into
//                    expert-contiguous rows, and the expert-sorted E4M3 terms
//                    of the normalised tokens (the gate/up GEMM's B operand);
//   combine_kernel   y = x + the token's weighted expert rows, in bf16.
#include <cfloat>
#include <climits>

#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// ----------------------------------------------------------------- route

// Top-k of one token's E logits (E <= 256) by one warp, then the softmax over
// the chosen (pnsm.cn overview, section 2.2): k rounds of a warp arg-max on
// (logit desc, index asc) -- ties go to the lower expert index; a NaN logit
// ranks below every number, so the k chosen indices are always distinct and
// in range.  `lg` may be shared or global memory.
__device__ __forceinline__ void topk_softmax_warp(const float *lg, int E, int k, int t, int *topk_idx, float *topk_w,
                                                  int lane) {
    float v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const int e = lane + 32 * c;
        const float l = e < E ? lg[e] : -INFINITY;
        v[c] = (l != l) ? -INFINITY : l;
    }
    unsigned taken = 0;
    float sel_l[8];
    int sel_e[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        if (r >= k) break;
        float bv = -INFINITY;
        int be = INT_MAX;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int e = lane + 32 * c;
            if (e < E && !((taken >> c) & 1u) && (v[c] > bv || (v[c] == bv && e < be))) {
                bv = v[c];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        sel_l[r] = bv;
        sel_e[r] = be;
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
    }
    if (lane == 0) {
        const float m = sel_l[0];
        float wsum = 0.f;
        float wv[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            if (r < k) {
                wv[r] = expf(sel_l[r] - m);
                wsum += wv[r];
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            if (r < k) {
                topk_idx[(size_t)t * k + r] = sel_e[r];
                topk_w[(size_t)t * k + r] = wv[r] / wsum;
            }
        }
    }
}

// ------------------------------------------- route, eight tokens per CTA
//
// One CTA per RF_TOK = 8 tokens, 8 warps.  Warp w normalises token w: the
// row's bf16 elements (8 per lane and load, up to RF_CHUNKS loads of a lane in
// flight), the sum of squares, 1/rms = 1/sqrt(mean(x^2) + eps) ("gpt-oss-20B"
// hub page, section 3.2); x_j scale_j -- exact in fp32, a product of two bf16
// numbers -- goes to shared memory, and xn_j = (x_j scale_j) (1/rms), rounded
// once, to global memory for the experts.  Router (same page, 3.4):
// logit_e = (1/rms) sum_j (x_j scale_j) W_r[e, j] + b_e, every product exact
// and the sum in fp32.  Warp w takes the tile of 4 tokens (4 (w / 4) ..) and
// 8 experts (groups w % 4, w % 4 + 4, ...); lane l the 4-element K chunks l,
// l + 32, ... of the row; packed fp32x2 FMAs sum each (token, expert) pair's
// even and odd elements in the two halves of one register pair.  A
// transposing warp reduction leaves the total of tile entry 8t + e in lane
// 8t + e.  Then the top-k and the softmax over the chosen, one warp per token.
constexpr int RF_TOK = 8;
constexpr int RF_THREADS = 256;
constexpr int RF_CHUNKS = 12;           // 8-element chunks of a row per lane and batch

__device__ __forceinline__ unsigned long long f32x2_pack(float lo, float hi) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(unsigned long long v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// two independent fp32 FMAs, each rounded once: (a.lo b.lo + c.lo, a.hi b.hi + c.hi)
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// bf16 pair (element j in the low half) -> fp32 pair
__device__ __forceinline__ unsigned long long bf16x2_to_f32x2(uint32_t w) {
    return f32x2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__global__ void __launch_bounds__(RF_THREADS, 2) route_fma_kernel(const RouteParams p) {
    extern __shared__ float rf_sm[];
    const int d = p.d, E = p.E;
    float *xs = rf_sm;                       // [RF_TOK][d] x * scale
    float *lg = xs + RF_TOK * d;             // [RF_TOK][E] logits
    float *rinv = lg + RF_TOK * E;           // [RF_TOK] 1/rms
    const int t0 = blockIdx.x * RF_TOK;
    const int ntok = min(RF_TOK, p.T - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();

    // ---- RMSNorm: warp w, token t0 + w
    {
        float *xr = xs + warp * d;
        const int nch = d / 8;
        if (warp < ntok) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (size_t)(t0 + warp) * d);
            const uint4 *scp = reinterpret_cast<const uint4 *>(p.norm_scale);
            float ss = 0.f;
            for (int c0 = 0; c0 < nch; c0 += 32 * RF_CHUNKS) {
                uint4 xv[RF_CHUNKS];
#pragma unroll
                for (int i = 0; i < RF_CHUNKS; ++i) {
                    const int c = c0 + lane + 32 * i;
                    xv[i] = c < nch ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int i = 0; i < RF_CHUNKS; ++i) {
                    const int c = c0 + lane + 32 * i;
                    if (c < nch) {
                        float f[8], sc[8];
                        bf16x8_to_f32(xv[i], f);
                        bf16x8_to_f32(__ldg(scp + c), sc);
#pragma unroll
                        for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
                        float4 *o = reinterpret_cast<float4 *>(xr + 8 * c);
                        o[0] = make_float4(f[0] * sc[0], f[1] * sc[1], f[2] * sc[2], f[3] * sc[3]);
                        o[1] = make_float4(f[4] * sc[4], f[5] * sc[5], f[6] * sc[6], f[7] * sc[7]);
                    }
                }
            }
            ss = warp_sum(ss);
            const float r = 1.0f / sqrtf(ss / (float)d + p.eps);
            if (lane == 0) rinv[warp] = r;
            __syncwarp();
            float4 *xo = reinterpret_cast<float4 *>(p.xn + (size_t)(t0 + warp) * d);
            const float4 *xi = reinterpret_cast<const float4 *>(xr);
            for (int c = lane; c < d / 4; c += 32) {
                const float4 v = xi[c];
                xo[c] = make_float4(v.x * r, v.y * r, v.z * r, v.w * r);
            }
        } else {
            for (int c = lane; c < d / 4; c += 32) reinterpret_cast<float4 *>(xr)[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane == 0) rinv[warp] = 0.f;
        }
    }
    __syncthreads();

    // ---- router logits: tile of 4 tokens x 8 experts per warp
    {
        const int tg = warp >> 2;
        const int n_eg = (E + 7) / 8;
        const float *xt = xs + (4 * tg) * d;
        for (int eg = warp & 3; eg < n_eg; eg += 4) {
            const int e0 = 8 * eg;
            unsigned long long acc[4][8];
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[t][e] = 0ull;
            // the router rows' chunk j of this group (zeros past the last expert)
            const uint2 *wbase = reinterpret_cast<const uint2 *>(p.router_w + (size_t)e0 * d);
            const int wstride = d / 4;              // uint2 per router row
            const int n_e = min(8, E - e0);
            for (int j = 4 * lane; j < d; j += 128) {
                uint2 wv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) wv[e] = e < n_e ? __ldg(wbase + e * wstride + (j >> 2)) : make_uint2(0, 0);
                ulonglong2 xv[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) xv[t] = *reinterpret_cast<const ulonglong2 *>(xt + t * d + j);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const unsigned long long w01 = bf16x2_to_f32x2(wv[e].x);
                    const unsigned long long w23 = bf16x2_to_f32x2(wv[e].y);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        acc[t][e] = ffma2(xv[t].x, w01, acc[t][e]);
                        acc[t][e] = ffma2(xv[t].y, w23, acc[t][e]);
                    }
                }
            }
            // entry 8t + e: the even and odd partial sums, then the sum over the lanes
            float v[32];
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float a, b;
                    f32x2_unpack(acc[t][e], a, b);
                    v[8 * t + e] = a + b;
                }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const bool upper = (lane & o) != 0;
#pragma unroll
                for (int i = 0; i < o; ++i) {
                    const float send = upper ? v[i] : v[i + o];
                    const float keep = upper ? v[i + o] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            const int tok = 4 * tg + (lane >> 3), e = e0 + (lane & 7);
            if (tok < ntok && e < E) lg[tok * E + e] = v[0] * rinv[tok] + p.router_b[e];
        }
    }
    __syncthreads();

    // ---- top-k and softmax, one warp per token
    if (warp < ntok) topk_softmax_warp(lg + warp * E, E, p.k, t0 + warp, p.topk_idx, p.topk_w, lane);
}

// ------------------------------------------------------ route, decode-sized
//
// Grid (token t, group of 16 experts); 16 warps, warp w owns expert 16y + w.
// Each warp loads its expert's router row into registers before anything
// else (the loads overlap the RMSNorm), every CTA normalises its token
// (RMSNorm as above, the same fp32 arithmetic), each warp writes one fp32
// logit, and the last CTA of the token to finish (a per-token counter, reset
// by that CTA) takes the top-k and the softmax.  CTA y = 0 writes xn.
constexpr int ROUTE_SMALL_CHUNKS = 12;   // 8-element chunks of a router row per lane: d <= 3072

__global__ void __launch_bounds__(512) route_small_kernel(const RouteParams p) {
    __shared__ float xs[ROUTE_SMALL_CHUNKS * 256];
    __shared__ float red[16];
    __shared__ int is_last;
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = p.d, E = p.E;
    const int e = blockIdx.y * 16 + warp;
    const int nch = d / 8;                   // 8-element chunks of a row
    uint4 wv[ROUTE_SMALL_CHUNKS];
#pragma unroll
    for (int i = 0; i < ROUTE_SMALL_CHUNKS; ++i) {
        const int c = lane + 32 * i;
        wv[i] = (e < E && c < nch) ? __ldg(reinterpret_cast<const uint4 *>(p.router_w + (size_t)e * d) + c)
                                   : make_uint4(0, 0, 0, 0);
    }
    // x may be the previous kernel's output: wait for it (the router rows above
    // are weights, never written by a kernel)
    pdl_wait();
    pdl_trigger();
    // RMSNorm: thread u owns chunks u and u + 512
    float f[2][8], sc[2][8];
    float ss = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = threadIdx.x + 512 * h;
        if (c < nch) {
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)t * d) + c), f[h]);
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(p.norm_scale) + c), sc[h]);
#pragma unroll
            for (int k = 0; k < 8; ++k) ss += f[h][k] * f[h][k];
        }
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) tot += red[i];
    const float inv_rms = 1.0f / sqrtf(tot / (float)d + p.eps);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = threadIdx.x + 512 * h;
        if (c < nch) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float v = f[h][k] * inv_rms * sc[h][k];
                f[h][k] = v;
                xs[8 * c + k] = v;
            }
            if (blockIdx.y == 0) {
                float4 *xo = reinterpret_cast<float4 *>(p.xn + (size_t)t * d + 8 * c);
                xo[0] = make_float4(f[h][0], f[h][1], f[h][2], f[h][3]);
                xo[1] = make_float4(f[h][4], f[h][5], f[h][6], f[h][7]);
            }
        }
    }
    __syncthreads();
    // logit of expert e
    if (e < E) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < ROUTE_SMALL_CHUNKS; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                float w8[8];
                bf16x8_to_f32(wv[i], w8);
                const float4 a = *reinterpret_cast<const float4 *>(xs + 8 * c);
                const float4 b = *reinterpret_cast<const float4 *>(xs + 8 * c + 4);
                acc = fmaf(a.x, w8[0], acc);
                acc = fmaf(a.y, w8[1], acc);
                acc = fmaf(a.z, w8[2], acc);
                acc = fmaf(a.w, w8[3], acc);
                acc = fmaf(b.x, w8[4], acc);
                acc = fmaf(b.y, w8[5], acc);
                acc = fmaf(b.z, w8[6], acc);
                acc = fmaf(b.w, w8[7], acc);
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) {
            p.logits[(size_t)t * E + e] = acc + p.router_b[e];
            __threadfence();
        }
    }
    // the token's last CTA takes the top-k
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&p.tok_done[t], 1u);
        is_last = prev == gridDim.y - 1;
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (warp == 0) {
        float lg[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int ee = lane + 32 * c;
            lg[c] = ee < E ? __ldcg(p.logits + (size_t)t * E + ee) : 0.f;
        }
        // stage the logits in shared memory for the warp arg-max
        float *lgs = xs;
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (lane + 32 * c < E) lgs[lane + 32 * c] = lg[c];
        __syncwarp();
        topk_softmax_warp(lgs, E, p.k, t, p.topk_idx, p.topk_w, lane);
        if (lane == 0) p.tok_done[t] = 0;
    }
}

// ------------------------------------------------------- group + permute
//
// Grid of G CTAs of 32 warps.  Every CTA computes the whole grouping of the
// P = T*k pairs (pair i = token i/k, slot i%k) in shared memory: warp w owns
// a contiguous segment of the pairs; pass 1 counts, per warp and expert, with
// __match_any_sync; a column scan turns the per-warp counts into each warp's
// starting position inside every expert's range; pass 2 assigns positions in
// pair order.  The result is sorted by expert and, within an expert, by token.
// CTA c then owns the expert-sorted rows [c*R, (c+1)*R): it writes their
// row_token / row_w / pair_row entries and their B operand row (below).  CTA 0
// writes counts, offsets and tiles.
//
// B operand row r: the normalised activations v = xn (fp32) of token
// row_token[r], as three E4M3 terms per 32-element block with E8M0 scale s
// (the exponent that fits the block maximum to 448):
//   hi = e4m3(v / 2^s),  lo = e4m3((v - hi 2^s) / 2^(s-4)),
//   lo2 = e4m3((v - hi 2^s - lo 2^(s-4)) / 2^s)
// (every residual is exact in fp32).  Out: xq[plane][r][0:Kd] (planes hi, lo,
// lo2; columns d..Kd zero) and xsf[g][plane][r] = the scale bytes of the
// 32-blocks 4g..4g+3 (byte i is block 4g+i) of plane 0 (hi, and lo2, which
// shares its scale) and plane 1 (lo).  A warp takes 32 consecutive 32-blocks of
// a row, one per lane.
constexpr int GROUP_ROWS_MAX = 1024;   // expert-sorted rows per CTA, at most

// Blocks b0 + lane (lane < 32) of token tok's encoding, written to the n_rows
// expert-sorted rows rows[0..n_rows) (the token's rows; n_rows <= 8).
__device__ __forceinline__ void quant_rows_part(const GroupParams &p, const int (&rows)[8], int n_rows, int tok, int b0,
                                                int lane) {
    const float4 *src = reinterpret_cast<const float4 *>(p.xn + (size_t)tok * p.d);
    const int nblk = p.d / 32, nblk_pad = p.Kd / 32;
    {
        const int b = b0 + lane;
        uint32_t s_hi = 127, s_lo = 127;
        uint32_t qh[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ql[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        uint32_t ql2[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (b < nblk) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 u = src[8 * b + i];
                v[4 * i] = u.x;
                v[4 * i + 1] = u.y;
                v[4 * i + 2] = u.z;
                v[4 * i + 3] = u.w;
            }
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
            const int e_hi = e4m3_block_exp(amax);
            const int e_lo = max(e_hi - 4, -126);
            const float inv_hi = pow2f(-e_hi), inv_lo = pow2f(-e_lo), mul_hi = pow2f(e_hi), mul_lo = pow2f(e_lo);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t h = f32x2_to_e4m3x2(v[2 * i] * inv_hi, v[2 * i + 1] * inv_hi);
                float d0, d1;
                e4m3x2_to_f32x2(h, d0, d1);
                const float r0 = v[2 * i] - d0 * mul_hi, r1 = v[2 * i + 1] - d1 * mul_hi;
                const uint32_t l = f32x2_to_e4m3x2(r0 * inv_lo, r1 * inv_lo);
                float l0, l1;
                e4m3x2_to_f32x2(l, l0, l1);
                const uint32_t l2 = f32x2_to_e4m3x2((r0 - l0 * mul_lo) * inv_hi, (r1 - l1 * mul_lo) * inv_hi);
                qh[i >> 1] |= h << (16 * (i & 1));
                ql[i >> 1] |= l << (16 * (i & 1));
                ql2[i >> 1] |= l2 << (16 * (i & 1));
            }
            s_hi = (uint32_t)(e_hi + 127);
            s_lo = (uint32_t)(e_lo + 127);
        }
        if (b < nblk_pad) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (q >= n_rows) break;
                const int r = rows[q];
                uint4 *dh = reinterpret_cast<uint4 *>(p.xq + (size_t)r * p.Kd + 32 * b);
                uint4 *dl = reinterpret_cast<uint4 *>(p.xq + ((size_t)p.P_max + r) * p.Kd + 32 * b);
                uint4 *dl2 = reinterpret_cast<uint4 *>(p.xq + ((size_t)2 * p.P_max + r) * p.Kd + 32 * b);
                dh[0] = make_uint4(qh[0], qh[1], qh[2], qh[3]);
                dh[1] = make_uint4(qh[4], qh[5], qh[6], qh[7]);
                dl[0] = make_uint4(ql[0], ql[1], ql[2], ql[3]);
                dl[1] = make_uint4(ql[4], ql[5], ql[6], ql[7]);
                dl2[0] = make_uint4(ql2[0], ql2[1], ql2[2], ql2[3]);
                dl2[1] = make_uint4(ql2[4], ql2[5], ql2[6], ql2[7]);
            }
        }
        // the scale bytes of four consecutive blocks (lanes 4m..4m+3) as one word
        uint32_t wh = s_hi, wl = s_lo;
#pragma unroll
        for (int i = 1; i < 4; ++i) {
            wh |= __shfl_down_sync(0xffffffffu, s_hi, i) << (8 * i);
            wl |= __shfl_down_sync(0xffffffffu, s_lo, i) << (8 * i);
        }
        if ((lane & 3) == 0 && b < nblk_pad) {
            const size_t g = (size_t)(b >> 2);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (q >= n_rows) break;
                p.xsf[(g * 2) * p.P_max + rows[q]] = wh;
                p.xsf[(g * 2 + 1) * p.P_max + rows[q]] = wl;
            }
        }
    }
}

template <bool QUANT>
__global__ void __launch_bounds__(1024) group_permute_kernel(const GroupParams p) {
    __shared__ int wcnt[32][257];
    __shared__ int off_s[257];
    __shared__ int tok_s[GROUP_ROWS_MAX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E, P = p.P;
    const int rows_per = (P + gridDim.x - 1) / gridDim.x;
    const int r0 = blockIdx.x * rows_per, r1 = min(P, r0 + rows_per);
    for (int i = threadIdx.x; i < 32 * 257; i += blockDim.x) (&wcnt[0][0])[i] = 0;
    pdl_wait();
    pdl_trigger();
    // the fused decode GEMM's per-token-block counters start at zero (after the wait: the
    // previous layer step's GEMM has finished with them)
    if (blockIdx.x == 0 && p.h_ready)
        for (int i = threadIdx.x; i < p.n_h_ready; i += blockDim.x) p.h_ready[i] = 0u;
    __syncthreads();
    const int seg = (P + 31) / 32;
    const int beg = warp * seg, end = min(P, beg + seg);

    // pass 1: per-warp counts; eight rows of 32 pairs are loaded before they are counted
    for (int base = beg; base < end; base += 256) {
        int ev[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = base + 32 * r + lane;
            ev[r] = i < end ? p.topk_idx[i] : -1;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = base + 32 * r + lane;
            int e = ev[r];
            if (i < end && (e < 0 || e >= E)) {
                if (blockIdx.x == 0) atomicOr(p.err, ERR_ROUTING);
                e = -1;
            }
            const unsigned m = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(m) - 1) wcnt[warp][e] += __popc(m);
            __syncwarp();
        }
    }
    __syncthreads();

    if ((int)threadIdx.x < E) {
        const int e = threadIdx.x;
        int s = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = wcnt[w][e];
            wcnt[w][e] = s;
            s += c;
        }
        if (blockIdx.x == 0) p.counts[e] = s;
        off_s[e] = s;   // total for now
    }
    __syncthreads();

    if (warp == 0) {
        // exclusive scans of counts and of token blocks; lane owns 8 experts
        int cnt[8], blk[8];
        int cs = 0, bs = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int e = lane * 8 + c;
            cnt[c] = e < E ? off_s[e] : 0;
            blk[c] = (cnt[c] + p.nb_rows - 1) / p.nb_rows;
            cs += cnt[c];
            bs += blk[c];
        }
        int ci = cs, bi = bs;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, ci, o);
            const int b = __shfl_up_sync(0xffffffffu, bi, o);
            if (lane >= o) {
                ci += a;
                bi += b;
            }
        }
        int co = ci - cs, bo = bi - bs;   // exclusive
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int e = lane * 8 + c;
            if (e < E) {
                off_s[e] = co;
                if (blockIdx.x == 0) {
                    p.offsets[e] = co;
                    p.tiles[e] = bo;
                }
            }
            co += cnt[c];
            bo += blk[c];
        }
        if (lane == 31 && blockIdx.x == 0) {
            p.offsets[E] = ci;
            p.tiles[E] = bi;
        }
    }
    __syncthreads();

    // pass 2: positions, in pair order within each warp's segment; this CTA keeps its rows
    for (int base = beg; base < end; base += 256) {
        int ev[8];
        float wv[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = base + 32 * r + lane;
            ev[r] = i < end ? p.topk_idx[i] : -1;
            wv[r] = i < end ? p.topk_w[i] : 0.f;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = base + 32 * r + lane;
            int e = ev[r];
            if (e >= E) e = -1;
            const unsigned m = __match_any_sync(0xffffffffu, e);
            if (e >= 0) {
                const int pos = off_s[e] + wcnt[warp][e] + __popc(m & ((1u << lane) - 1u));
                if (pos >= r0 && pos < r1) {
                    p.row_token[pos] = i / p.k;
                    p.row_w[pos] = wv[r];
                    p.pair_row[i] = pos;
                    tok_s[pos - r0] = i / p.k;
                }
            }
            __syncwarp();
            if (e >= 0 && lane == __ffs(m) - 1) wcnt[warp][e] += __popc(m);
            __syncwarp();
        }
    }
    if constexpr (QUANT) {
        __syncthreads();
        // this CTA's rows of the B operand: one warp per (row, 32 blocks of 32 elements), so
        // that a row's loads are spread over warps rather than chained in one
        const int parts = (p.Kd / 32 + 31) / 32;
        for (int u = warp; u < (r1 - r0) * parts; u += 32) {
            const int rr = u / parts;
            const int rows[8] = {r0 + rr, 0, 0, 0, 0, 0, 0, 0};
            quant_rows_part(p, rows, 1, tok_s[rr], (u - rr * parts) * 32, lane);
        }
    }
}

// Large batches: the B operand token by token, after the grouping kernel.  A
// warp takes (token, 32 blocks of 32 elements): it reads the token's normalised
// row once, encodes it once and writes it to the token's k expert-sorted rows
// (pair_row), so every token is read once rather than k times.
__global__ void __launch_bounds__(256) encode_tokens_kernel(const GroupParams p, int T) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int parts = (p.Kd / 32 + 31) / 32;
    const long long n_tasks = (long long)T * parts;
    const long long n_warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long u = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < n_tasks; u += n_warps) {
        const int tok = (int)(u / parts), part = (int)(u % parts);
        const int mine = lane < p.k ? __ldg(p.pair_row + (size_t)tok * p.k + lane) : 0;
        int rows[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) rows[q] = __shfl_sync(0xffffffffu, mine, q);
        quant_rows_part(p, rows, p.k, tok, part * 32, lane);
    }
}

// ------------------------------- route and group, decode-sized, one launch
//
// T <= RGS_MAX_T tokens: a CTA per token, 16 warps.  The token's RMSNorm and its
// E logits take route_small_kernel's arithmetic (the same values), warp w taking
// experts w, w + 16, ...; then the top-k and the softmax over the chosen, and xn
// to global memory.  A grid-wide barrier follows: a counter the last CTA to
// arrive resets and a generation word it then advances, with a bounded wait (a
// CTA per token fits the GPU in one wave, so every CTA is resident before any
// waits for long).  After it every CTA computes the grouping of all T k pairs in
// shared memory, in group_permute_kernel's stable order (by expert, then pair):
// per-warp match counts, a scan over warps, a scan over experts.  CTA 0 writes
// counts, offsets and tiles; each CTA writes its own token's k pairs -- their
// row_token, row_w and pair_row entries -- and the three E4M3 planes of its xn
// into those k rows (quant_rows_part).  The outputs equal those of
// route_small_kernel followed by group_permute_kernel, bit for bit.
constexpr int RGS_MAX_T = 64;

__global__ void __launch_bounds__(512) route_group_small_kernel(const RouteParams rp, const GroupParams gp,
                                                                unsigned int *bar, unsigned long long wait_limit_ns) {
    __shared__ float xs[ROUTE_SMALL_CHUNKS * 256];
    __shared__ float red[16];
    __shared__ float lg[256];
    __shared__ int wcnt[16][257];
    __shared__ int off_s[257];
    __shared__ int pos_s[8];
    __shared__ int go_s;
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = rp.d, E = rp.E, k = rp.k;
    const int nch = d / 8;
    for (int i = threadIdx.x; i < 16 * 257; i += blockDim.x) (&wcnt[0][0])[i] = 0;
    if (threadIdx.x < 8) pos_s[threadIdx.x] = -1;
    pdl_wait();
    pdl_trigger();
    // the fused decode GEMM's per-token-block counters start at zero (it runs after this
    // launch; the wait above orders this after the previous layer step's GEMM)
    if (t == 0 && gp.h_ready)
        for (int i = threadIdx.x; i < gp.n_h_ready; i += blockDim.x) gp.h_ready[i] = 0u;

    // ---- RMSNorm of token t (route_small_kernel's arithmetic): thread u owns chunks u and u + 512
    float f[2][8], sc[2][8];
    float ss = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = threadIdx.x + 512 * h;
        if (c < nch) {
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(rp.x + (size_t)t * d) + c), f[h]);
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(rp.norm_scale) + c), sc[h]);
#pragma unroll
            for (int q = 0; q < 8; ++q) ss += f[h][q] * f[h][q];
        }
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) tot += red[i];
    const float inv_rms = 1.0f / sqrtf(tot / (float)d + rp.eps);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = threadIdx.x + 512 * h;
        if (c < nch) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float v = f[h][q] * inv_rms * sc[h][q];
                f[h][q] = v;
                xs[8 * c + q] = v;
            }
            float4 *xo = reinterpret_cast<float4 *>(rp.xn + (size_t)t * d + 8 * c);
            xo[0] = make_float4(f[h][0], f[h][1], f[h][2], f[h][3]);
            xo[1] = make_float4(f[h][4], f[h][5], f[h][6], f[h][7]);
        }
    }
    __syncthreads();

    // ---- logits of experts warp, warp + 16, ... (route_small_kernel's per-warp sum)
    for (int e = warp; e < E; e += 16) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < ROUTE_SMALL_CHUNKS; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                float w8[8];
                bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(rp.router_w + (size_t)e * d) + c), w8);
                const float4 a = *reinterpret_cast<const float4 *>(xs + 8 * c);
                const float4 b = *reinterpret_cast<const float4 *>(xs + 8 * c + 4);
                acc = fmaf(a.x, w8[0], acc);
                acc = fmaf(a.y, w8[1], acc);
                acc = fmaf(a.z, w8[2], acc);
                acc = fmaf(a.w, w8[3], acc);
                acc = fmaf(b.x, w8[4], acc);
                acc = fmaf(b.y, w8[5], acc);
                acc = fmaf(b.z, w8[6], acc);
                acc = fmaf(b.w, w8[7], acc);
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) lg[e] = acc + rp.router_b[e];
    }
    __syncthreads();
    if (warp == 0) topk_softmax_warp(lg, E, k, t, rp.topk_idx, rp.topk_w, lane);

    // ---- grid-wide barrier: every token's top-k (and xn) written
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned int gen = ld_acquire_gpu(bar + 1);    // before arriving: the last arrival advances it
        const unsigned int n = atomicAdd(bar, 1u);
        int ok = 1;
        if (n == gridDim.x - 1) {
            atomicExch(bar, 0u);
            __threadfence();
            atomicAdd(bar + 1, 1u);
        } else {
            const uint64_t start = globaltimer_ns();
            while (ld_acquire_gpu(bar + 1) == gen) {
                if (globaltimer_ns() - start > wait_limit_ns) {
                    atomicOr(gp.err, ERR_WAIT_ROUTE);
                    ok = 0;
                    break;
                }
            }
        }
        __threadfence();
        go_s = ok;
    }
    __syncthreads();
    if (!go_s) return;

    // ---- the grouping of all P pairs (pair i = token i / k, slot i % k), one pair per thread
    const int P = gp.P;
    const int i = threadIdx.x;
    int e_i = -1;
    if (i < P) {
        e_i = __ldcg(gp.topk_idx + i);
        if (e_i < 0 || e_i >= E) {
            if (t == 0) atomicOr(gp.err, ERR_ROUTING);
            e_i = -1;
        }
    }
    const unsigned m = __match_any_sync(0xffffffffu, e_i);
    if (e_i >= 0 && lane == __ffs(m) - 1) wcnt[warp][e_i] = __popc(m);
    __syncthreads();
    if ((int)threadIdx.x < E) {
        const int e = threadIdx.x;
        int s = 0;
        for (int w = 0; w < 16; ++w) {
            const int c = wcnt[w][e];
            wcnt[w][e] = s;
            s += c;
        }
        if (t == 0) gp.counts[e] = s;
        off_s[e] = s;   // total for now
    }
    __syncthreads();
    if (warp == 0) {
        // exclusive scans of counts and of token blocks; lane owns 8 experts
        int cnt[8], blk[8];
        int cs = 0, bs = 0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int e = lane * 8 + c;
            cnt[c] = e < E ? off_s[e] : 0;
            blk[c] = (cnt[c] + gp.nb_rows - 1) / gp.nb_rows;
            cs += cnt[c];
            bs += blk[c];
        }
        int ci = cs, bi = bs;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, ci, o);
            const int b = __shfl_up_sync(0xffffffffu, bi, o);
            if (lane >= o) {
                ci += a;
                bi += b;
            }
        }
        int co = ci - cs, bo = bi - bs;   // exclusive
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int e = lane * 8 + c;
            if (e < E) {
                off_s[e] = co;
                if (t == 0) {
                    gp.offsets[e] = co;
                    gp.tiles[e] = bo;
                }
            }
            co += cnt[c];
            bo += blk[c];
        }
        if (lane == 31 && t == 0) {
            gp.offsets[E] = ci;
            gp.tiles[E] = bi;
        }
    }
    __syncthreads();
    // this token's pairs: their rows and permutation entries
    if (e_i >= 0 && i >= t * k && i < t * k + k) {
        const int pos = off_s[e_i] + wcnt[warp][e_i] + __popc(m & ((1u << lane) - 1u));
        pos_s[i - t * k] = pos;
        gp.row_token[pos] = t;
        gp.row_w[pos] = __ldcg(gp.topk_w + i);
        gp.pair_row[i] = pos;
    }
    __syncthreads();
    // the token's three E4M3 planes into its k rows, a warp per 32 blocks of 32 elements
    const int parts = (gp.Kd / 32 + 31) / 32;
    if (warp < parts) {
        int rows[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        int n_rows = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (q < k && pos_s[q] >= 0) rows[n_rows++] = pos_s[q];
        quant_rows_part(gp, rows, n_rows, t, warp * 32, lane);
    }
}

// --------------------------------------------------------------- combine
//
// y[t] = bf16(x[t] + sum_i o[pair_row[t*k + i]]) in fp32, the k weighted
// expert rows added in the token's slot order (descending router logit), so
// the result does not depend on scheduling.  Each thread handles 8
// consecutive features of one token.
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t *__restrict__ x, const float *__restrict__ orows,
                                                      const int *__restrict__ pair_row, uint16_t *__restrict__ y,
                                                      int T, int d, int k) {
    const int per_tok = d / 8;
    const long long n = (long long)T * per_tok;
    // x (the block's input) and pair_row (from the group kernel, which finished before
    // the GEMMs started) are final before this kernel launches: the first unit's
    // loads of them go out before the wait for the down GEMM's rows
    long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    uint4 xv = make_uint4(0, 0, 0, 0);
    int prow[8];
    if (i < n) {
        const int t = (int)(i / per_tok), j = (int)(i % per_tok) * 8;
        xv = *reinterpret_cast<const uint4 *>(x + (size_t)t * d + j);
#pragma unroll
        for (int s = 0; s < 8; ++s) prow[s] = s < k ? __ldcg(pair_row + (size_t)t * k + s) : 0;
    }
    pdl_wait();
    pdl_trigger();
    for (bool first = true; i < n; i += (long long)gridDim.x * blockDim.x, first = false) {
        const int t = (int)(i / per_tok), j = (int)(i % per_tok) * 8;
        float acc[8];
        if (!first) {
            xv = *reinterpret_cast<const uint4 *>(x + (size_t)t * d + j);
#pragma unroll
            for (int s = 0; s < 8; ++s) prow[s] = s < k ? pair_row[(size_t)t * k + s] : 0;
        }
        bf16x8_to_f32(xv, acc);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            if (s >= k) break;
            const float4 *o = reinterpret_cast<const float4 *>(orows + (size_t)prow[s] * d + j);
            const float4 a = o[0], b = o[1];
            acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
            acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
        }
        const __nv_bfloat162 p0 = __floats2bfloat162_rn(acc[0], acc[1]), p1 = __floats2bfloat162_rn(acc[2], acc[3]);
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(acc[4], acc[5]), p3 = __floats2bfloat162_rn(acc[6], acc[7]);
        uint4 out;
        out.x = *reinterpret_cast<const uint32_t *>(&p0);
        out.y = *reinterpret_cast<const uint32_t *>(&p1);
        out.z = *reinterpret_cast<const uint32_t *>(&p2);
        out.w = *reinterpret_cast<const uint32_t *>(&p3);
        *reinterpret_cast<uint4 *>(y + (size_t)t * d + j) = out;
    }
}

// ------------------------------------------------------------ debug decode
//
// The grouped GEMMs' weight decode on its own: one thread per (row, 32-element
// block); fp16 e2m1 conversion times the block multiplier under the row shift,
// then times 2^c back in fp32.
__global__ void decode_kernel(const uint8_t *codes, const uint8_t *scales, int R, int K, float *out) {
    const int nb = K / 32;
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (idx >= (long long)R * nb) return;
    const int r = (int)(idx / nb), b = (int)(idx % nb);
    const uint8_t *srow = scales + (size_t)r * nb;
    int smax = -1;
    for (int i = 0; i < nb; ++i)
        if (srow[i] != 255 && srow[i] > smax) smax = srow[i];
    const int c = row_shift_from_max(smax);
    const uint32_t mult = block_multiplier(srow[b], c);
    const float back = exp2i(c);
    const uint32_t *cw = reinterpret_cast<const uint32_t *>(codes + (size_t)r * (K / 2) + b * 16);
    float *o = out + (size_t)r * K + b * 32;
    for (int wi = 0; wi < 4; ++wi) {
        uint32_t h4[4];
        e2m1x8_to_half2x4(cw[wi], h4);
        for (int j = 0; j < 4; ++j) {
            const uint32_t v = hmul2_u32(h4[j], mult);
            const __half2 hv = *reinterpret_cast<const __half2 *>(&v);
            const float2 f = __half22float2(hv);
            o[wi * 8 + 2 * j] = f.x * back;
            o[wi * 8 + 2 * j + 1] = f.y * back;
        }
    }
}

// ----------------------------------------------------------- wait self-test

__global__ void selftest_wait_kernel(unsigned int *err, unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const WaitCtl wc{&abort_flag, err, ERR_WAIT_SELFTEST, limit_ns};
    // nothing ever arrives on `bar`: the wait must run out and report it
    (void)mbar_wait(&bar, 0, wc);
}

// --------------------------------------------------------------- launchers

cudaError_t launch_route(const RouteParams &p, cudaStream_t s) {
    if (p.T <= 0) return cudaSuccess;
    // decode-sized batches: a CTA per (token, 16 experts), router rows held in registers
    if (p.T <= 512 && p.d <= ROUTE_SMALL_CHUNKS * 256 && p.logits && p.tok_done) {
        return launch_pdl(route_small_kernel, dim3(p.T, (p.E + 15) / 16), dim3(512), 0, s, p);
    }
    // otherwise eight tokens per CTA, the router on CUDA cores (packed fp32x2 FMAs); at most
    // 8 (6144 + 256) + 8 floats = 200 KB of shared memory
    const size_t smem = ((size_t)RF_TOK * (p.d + p.E) + RF_TOK) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(route_fma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(route_fma_kernel, dim3((p.T + RF_TOK - 1) / RF_TOK), dim3(RF_THREADS), smem, s, p);
}

// Route and group of a decode-sized batch in one launch; false when the batch is
// not one (the caller then launches the two stages).
bool route_group_small_fits(const RouteParams &p) {
    return p.T >= 1 && p.T <= RGS_MAX_T && p.d <= ROUTE_SMALL_CHUNKS * 256 && p.E <= 256 && p.k <= 8;
}

cudaError_t launch_route_group_small(const RouteParams &rp, const GroupParams &gp, unsigned int *bar,
                                     unsigned long long wait_limit_ns, cudaStream_t s) {
    return launch_pdl(route_group_small_kernel, dim3(rp.T), dim3(512), 0, s, rp, gp, bar, wait_limit_ns);
}

// Pairs above which the grouping and the token-major encoding run as two kernels.
constexpr int GROUP_SPLIT_PAIRS = 2048;

cudaError_t launch_group(const GroupParams &p, cudaStream_t s) {
    if (p.P <= 0) return cudaSuccess;
    if (p.P <= GROUP_SPLIT_PAIRS) {
        // one kernel: a CTA per 8 rows, each encoding its own rows
        int grid = (p.P + 7) / 8;
        if (grid > 148) grid = 148;
        if ((p.P + grid - 1) / grid > GROUP_ROWS_MAX) grid = (p.P + GROUP_ROWS_MAX - 1) / GROUP_ROWS_MAX;
        return launch_pdl(group_permute_kernel<true>, dim3(grid), dim3(1024), 0, s, p);
    }
    // the grouping with up to GROUP_ROWS_MAX rows per CTA, then the tokens' encoding
    const int grid = (p.P + GROUP_ROWS_MAX - 1) / GROUP_ROWS_MAX;
    cudaError_t e = launch_pdl(group_permute_kernel<false>, dim3(grid), dim3(1024), 0, s, p);
    if (e != cudaSuccess) return e;
    const int T = p.P / p.k;
    const int parts = (p.Kd / 32 + 31) / 32;
    long long ctas = ((long long)T * parts + 7) / 8;
    if (ctas > 148 * 8) ctas = 148 * 8;
    return launch_pdl(encode_tokens_kernel, dim3((unsigned)ctas), dim3(256), 0, s, p, T);
}

cudaError_t launch_combine(const uint16_t *x, const float *orows, const int *pair_row, uint16_t *y, int T, int d, int k,
                           cudaStream_t s) {
    const long long n = (long long)T * (d / 8);
    if (n == 0) return cudaSuccess;
    const int grid = (int)min((n + 255) / 256, (long long)148 * 8);
    return launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, s, x, orows, pair_row, y, T, d, k);
}

cudaError_t launch_decode(const uint8_t *codes, const uint8_t *scales, int R, int K, float *out, cudaStream_t s) {
    const long long n = (long long)R * (K / 32);
    if (n == 0) return cudaSuccess;
    decode_kernel<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(codes, scales, R, K, out);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(unsigned int *err, unsigned long long limit_ns, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace moe
