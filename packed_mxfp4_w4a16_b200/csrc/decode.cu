// decode.cu — sm_100a kernels of the batch-1 decode path of the packed-MXFP4
// W4A16 top-4 MoE expert FFN:
//
//   route_kernel           router projection (+ optional weightless RMSNorm of a
//                          residual stream), then top-k + softmax by the last CTA
//                          of each token.
//   gateup_decode_kernel   fused gate and up packed GEMVs + SwiGLU, all selected
//                          (token, slot) pairs of the call in one launch.
//   down_decode_kernel     down packed GEMV of every slot + the sequential BF16
//                          routing-weighted combine (+ residual) in one launch.
//
// Sources (model card "LFM2.5-24B-A2B — Packed MXFP4 Inference"): section "What
// was optimized" > "Grouped top-4 expert execution" (grouped gate GEMV, grouped
// up GEMV, activation and multiplication, grouped down GEMV, fused combine that
// keeps sequential BF16 multiply/add rounding); "Direct reads from GPU-resident
// weights" (experts read in place through a device pointer table); "GPU routing
// inside resident-layer graphs" (projection, bias, top-k, coefficients on the
// GPU, no id copy to the host); table "Model and quantization" (E2M1 + E8M0 per
// 32, BF16 activations, FP32 accumulation, BF16 outputs).
//
// Memory plan.  Each GEMV CTA owns one SM (512 threads) and a contiguous range
// of output rows; a "team" of TL lanes streams one packed row with 16-byte
// non-allocating loads (one 16-byte chunk = one 32-element E8M0 group), two rows
// in flight per team.  Codes are decoded in registers by the E2M1->f16x2
// conversion instruction and multiplied with FP16-staged activations in FP32
// (fma.rn.f32.f16); each group's partial sum is scaled by its E8M0 exponent in
// FP32.  Team partial sums meet through warp shuffles.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.cuh"

namespace moe {

constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kDownWarps = kDownThreads / 32;

// ------------------------------------------------------------------ route --
// grid (E, ceil(T / 8)); warp w of CTA (e, b) computes logit[t = 8b + w][e].
// The router row is fetched before the programmatic-launch wait (it is a
// constant input), so its DRAM latency overlaps the previous kernel's tail.

constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kRouteMaxChunks = 16;  // H <= 16 * 32 * 8 = 4096 for the register path

__global__ void __launch_bounds__(kRouteThreads)
route_kernel(const RouteParams p) {
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x, H = p.H, E = p.E, k = p.k;
    const int t = blockIdx.y * kRouteWarps + warp;
    const int nch = H >> 3;  // 16-byte chunks of 8 BF16
    const bool active = t < p.T;

    uint4 wv[kRouteMaxChunks];
    const uint16_t *row = p.wr + (size_t)e * H;
#pragma unroll
    for (int m = 0; m < kRouteMaxChunks; ++m) {
        const int c = lane + 32 * m;
        wv[m] = (active && c < nch) ? *reinterpret_cast<const uint4 *>(row + (size_t)c * 8)
                                    : make_uint4(0u, 0u, 0u, 0u);
    }

    pdl_wait();
    pdl_launch_dependents();

    if (active) {
        const uint16_t *xt = p.x + (size_t)t * H;
        uint4 xv[kRouteMaxChunks];
        float ss = 0.f;
#pragma unroll
        for (int m = 0; m < kRouteMaxChunks; ++m) {
            const int c = lane + 32 * m;
            xv[m] = c < nch ? *reinterpret_cast<const uint4 *>(xt + (size_t)c * 8)
                            : make_uint4(0u, 0u, 0u, 0u);
            if (p.rmsnorm) {
                const uint32_t w4[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a = bf16_to_f32(w4[q] & 0xFFFFu), b = bf16_to_f32(w4[q] >> 16);
                    ss = fmaf(a, a, ss);
                    ss = fmaf(b, b, ss);
                }
            }
        }
        float inv = 1.f;
        if (p.rmsnorm) inv = 1.0f / sqrtf(warp_sum(ss) / (float)H + p.eps);
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < kRouteMaxChunks; ++m) {
            const int c = lane + 32 * m;
            if (c < nch) {
                uint32_t x4[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
                const uint32_t r4[4] = {wv[m].x, wv[m].y, wv[m].z, wv[m].w};
                if (p.rmsnorm) {
                    // weightless RMSNorm: xn = BF16(r / sqrt(mean(r^2) + eps))
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        x4[q] = (uint32_t)f32_to_bf16(bf16_to_f32(x4[q] & 0xFFFFu) * inv) |
                                ((uint32_t)f32_to_bf16(bf16_to_f32(x4[q] >> 16) * inv) << 16);
                    if (e == 0)
                        *reinterpret_cast<uint4 *>(p.x_norm + (size_t)t * H + (size_t)c * 8) =
                            make_uint4(x4[0], x4[1], x4[2], x4[3]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc = fmaf(bf16_to_f32(x4[q] & 0xFFFFu), bf16_to_f32(r4[q] & 0xFFFFu), acc);
                    acc = fmaf(bf16_to_f32(x4[q] >> 16), bf16_to_f32(r4[q] >> 16), acc);
                }
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) {
            if (p.bias) acc += p.bias[e];
            p.logits_ws[(size_t)t * E + e] = acc;
        }
    }

    // the last CTA of this token block selects; an arrival counter, no waiting
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(p.counters + blockIdx.y, 1u);
        s_last = (prev == (unsigned)E - 1u);
    }
    __syncthreads();
    if (!s_last || !active) return;
    __threadfence();

    // top-k of logits[t][0..E): ids descending, equal logits -> lower id.
    // Each round: warp-wide max of an order-preserving key of the logit, then
    // the minimum id among the lanes holding that key (two redux operations).
    const float *lg = p.logits_ws + (size_t)t * E;
    constexpr int kMaxPerLane = 32;  // E <= 1024
    const int per = (E + 31) >> 5;
    uint32_t key[kMaxPerLane];
#pragma unroll
    for (int m = 0; m < kMaxPerLane; ++m) {
        const int ee = lane + 32 * m;
        uint32_t kk = 0u;  // below every logit: never chosen
        if (m < per && ee < E) {
            const float v = __ldcg(lg + ee);
            const uint32_t b = __float_as_uint(v);
            kk = (v != v) ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
        }
        key[m] = kk;
    }
    int chosen[kMaxTopK];
    float chosen_v[kMaxTopK];
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int m = 0; m < kMaxPerLane; ++m)
            if (key[m] > bk) {  // ascending m: ties keep the lower id
                bk = key[m];
                bi = lane + 32 * m;
            }
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const int wi = (int)__reduce_min_sync(0xffffffffu, bk == wk ? (uint32_t)bi : 0x7FFFFFFFu);
        chosen[j] = wi;
        chosen_v[j] = __uint_as_float((wk & 0x80000000u) ? (wk & 0x7FFFFFFFu) : ~wk);
        if ((wi & 31) == lane && wi < E) {
#pragma unroll
            for (int m = 0; m < kMaxPerLane; ++m)
                if (m == (wi >> 5)) key[m] = 0u;
        }
    }
    if (lane == 0) {
        // coefficients: softmax over the k selected logits (slot 0 holds the max)
        float z = 0.f, ex[kMaxTopK];
        for (int j = 0; j < k; ++j) {
            ex[j] = expf(chosen_v[j] - chosen_v[0]);
            z += ex[j];
        }
        for (int j = 0; j < k; ++j) {
            p.ids[(size_t)t * k + j] = chosen[j];
            p.w[(size_t)t * k + j] = ex[j] / z;
        }
    }
    if (p.logits_out)
        for (int ee = lane; ee < E; ee += 32) p.logits_out[(size_t)t * E + ee] = __ldcg(lg + ee);
    if (warp == 0 && lane == 0) p.counters[blockIdx.y] = 0u;
}

// ------------------------------------------------------------- team tools --
// A "team" of TL lanes (TL a power of two, aligned in the warp) owns one packed
// row at a time; lane lt of the team holds the KCH consecutive 16-byte chunks
// [lt*KCH, lt*KCH + KCH) of the row (one E8M0 group each) and the matching
// FP16-staged activations in registers.  Teams are independent: their
// shuffles use the team's own lane mask.

template <int TL>
__device__ __forceinline__ unsigned team_mask(int lane) {
    return TL == 32 ? 0xffffffffu : (((1u << TL) - 1u) << (lane & ~(TL - 1)));
}

template <int TL>
__device__ __forceinline__ float team_max(float v, unsigned mask) {
#pragma unroll
    for (int o = TL / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(mask, v, o));
    return v;
}

template <int TL>
__device__ __forceinline__ float team_add(float v, unsigned mask) {
#pragma unroll
    for (int o = TL / 2; o > 0; o >>= 1) v += __shfl_xor_sync(mask, v, o);
    return v;
}

// Load this lane's part of BF16 vector v (K elements), stage it as FP16 words
// scaled by 2^-c where c comes from the team-wide max |v|; returns c.
template <int TL, int KCH>
__device__ __forceinline__ int stage_x(const uint16_t *v, int lt, int C, unsigned mask,
                                       uint32_t (&xw)[KCH][16]) {
    uint4 raw[KCH][4];
    float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < KCH; ++u) {
        const int c = lt * KCH + u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            raw[u][q] = c < C ? *reinterpret_cast<const uint4 *>(v + (size_t)c * 32 + q * 8)
                              : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w4[4] = {raw[u][q].x, raw[u][q].y, raw[u][q].z, raw[u][q].w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                m[i] = fmaxf(m[i], fmaxf(fabsf(bf16_to_f32(w4[i] & 0xFFFFu)),
                                         fabsf(bf16_to_f32(w4[i] >> 16))));
        }
    }
    const int c = f16_stage_exponent(team_max<TL>(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), mask));
    const float sf = pow2_neg(c);
#pragma unroll
    for (int u = 0; u < KCH; ++u)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t w4[4] = {raw[u][q].x, raw[u][q].y, raw[u][q].z, raw[u][q].w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                xw[u][q * 4 + i] = f32x2_to_f16x2(bf16_to_f32(w4[i] & 0xFFFFu) * sf,
                                                  bf16_to_f32(w4[i] >> 16) * sf);
        }
    return c;
}

template <int KCH>
__device__ __forceinline__ void load_chunks(const uint8_t *codes, const uint8_t *scales, bool ok,
                                            int lt, int C, uint4 (&cw)[KCH], uint32_t (&sc)[KCH]) {
#pragma unroll
    for (int u = 0; u < KCH; ++u) {
        const int c = lt * KCH + u;
        if (ok && c < C) {
            cw[u] = ld_stream16(codes + (size_t)c * 16);
            sc[u] = ld_stream_u8(scales + c);
        } else {
            cw[u] = make_uint4(0u, 0u, 0u, 0u);
            sc[u] = 127u;
        }
    }
}

template <int KCH>
__device__ __forceinline__ float chunks_dot(const uint4 (&cw)[KCH], const uint32_t (&sc)[KCH],
                                            const uint32_t (&xw)[KCH][16]) {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < KCH; ++u) {
        float a0 = 0.f, a1 = 0.f;
        dot8_e2m1_f16(cw[u].x, xw[u][0], xw[u][1], xw[u][2], xw[u][3], a0, a1);
        dot8_e2m1_f16(cw[u].y, xw[u][4], xw[u][5], xw[u][6], xw[u][7], a0, a1);
        dot8_e2m1_f16(cw[u].z, xw[u][8], xw[u][9], xw[u][10], xw[u][11], a0, a1);
        dot8_e2m1_f16(cw[u].w, xw[u][12], xw[u][13], xw[u][14], xw[u][15], a0, a1);
        acc = fmaf(a0 + a1, e8m0_to_f32(sc[u]), acc);
    }
    return acc;
}

// ----------------------------------------------------------- gate / up ----

// L2 prefetch of this CTA's slice of the selected experts' down matrices, so
// that the down GEMV that follows reads them from L2 while the DRAM keeps
// streaming.  One lane per (token, slot) pair; an expert chosen by several
// pairs is fetched by the lowest such lane only.  Slices are 16-byte multiples
// computed on the host (codes: pf_codes bytes, scales: pf_scales bytes).
__device__ __forceinline__ void prefetch_down_slice(const GateUpParams &p, int lane) {
    const int P = p.T * p.k;
    const int Pr = (P + 31) & ~31;  // every lane iterates the same number of times
    for (int q = lane; q < Pr; q += 32) {
        const int e = q < P ? p.ids[q] : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const bool leader = (__ffs(same) - 1) == lane;
        if (q < P && leader && e >= 0 && e < p.E) {
            const size_t mc = (size_t)p.H * p.I / 2, ms = (size_t)p.H * p.I / 32;
            const size_t oc = (size_t)blockIdx.x * p.pf_codes;
            const size_t os = (size_t)blockIdx.x * p.pf_scales;
            if (oc < mc) {
                const size_t n = min((size_t)p.pf_codes, mc - oc);
                prefetch_l2_bulk(p.table[e].codes[2] + oc, (uint32_t)n);
            }
            if (os < ms) {
                const size_t n = min((size_t)p.pf_scales, ms - os);
                prefetch_l2_bulk(p.table[e].scales[2] + os, (uint32_t)n);
            }
        }
    }
}

// Items are (pair q = t*k + j, row i), q-major; each team owns a contiguous
// range of items and processes two rows per step (gate and up of each).
template <int TL, int KCH>
__global__ void __launch_bounds__(kGemvThreads, 1)
gateup_decode_kernel(const GateUpParams p) {
    constexpr int TPW = 32 / TL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lt = lane & (TL - 1);
    const unsigned mask = team_mask<TL>(lane);
    const int H = p.H, I = p.I, k = p.k;
    const int C = H >> 5;
    const size_t rc = (size_t)H >> 1, rs = (size_t)H >> 5;  // bytes per row: codes, scales

    pdl_wait();  // x and ids come from earlier kernels
    pdl_launch_dependents();
    if (p.prefetch_down && warp == kGemvWarps - 1) prefetch_down_slice(p, lane);

    const long long N = (long long)p.T * k * I;
    const long long nteams = (long long)gridDim.x * kGemvWarps * TPW;
    const long long team = ((long long)blockIdx.x * kGemvWarps + warp) * TPW + (lane / TL);
    long long it = N * team / nteams;
    const long long end = N * (team + 1) / nteams;

    uint32_t xw[KCH][16];
    int cur_tok = -1, cur_q = -1;
    float xs = 1.f;
    bool bad = false;
    const uint8_t *gc = nullptr, *gs = nullptr, *uc = nullptr, *us = nullptr;

    while (it < end) {
        const int q = (int)(it / I);
        const int row = (int)(it - (long long)q * I);
        // a second row of the same pair in this step if there is one
        const bool two = (it + 1 < end) && (row + 1 < I);
        if (q != cur_q) {
            const int e = p.ids[q];
            bad = (e < 0 || e >= p.E);
            if (!bad) {
                const ExpertPtrs *ep = p.table + e;
                gc = ep->codes[0];
                gs = ep->scales[0];
                uc = ep->codes[1];
                us = ep->scales[1];
            }
            cur_q = q;
        }
        uint4 cg[2][KCH], cu[2][KCH];
        uint32_t sg[2][KCH], su[2][KCH];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const bool ok = !bad && (u == 0 || two);
            const size_t r = (size_t)(row + u);
            load_chunks<KCH>(gc + r * rc, gs + r * rs, ok, lt, C, cg[u], sg[u]);
            load_chunks<KCH>(uc + r * rc, us + r * rs, ok, lt, C, cu[u], su[u]);
        }
        const int tok = q / k;
        if (tok != cur_tok) {
            xs = pow2(stage_x<TL, KCH>(p.x + (size_t)tok * H, lt, C, mask, xw));
            cur_tok = tok;
        }
        float v[4];
        v[0] = chunks_dot<KCH>(cg[0], sg[0], xw);
        v[1] = chunks_dot<KCH>(cu[0], su[0], xw);
        v[2] = chunks_dot<KCH>(cg[1], sg[1], xw);
        v[3] = chunks_dot<KCH>(cu[1], su[1], xw);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = team_add<TL>(v[i], mask);
        if (lt < 2 && (lt == 0 || two)) {
            const float ag = lt == 0 ? v[0] : v[2];
            const float au = lt == 0 ? v[1] : v[3];
            uint16_t out = 0;
            if (!bad) {
                const float g = round_bf16(ag * xs);
                const float uu = round_bf16(au * xs);
                const float s = round_bf16(g / (1.0f + expf(-g)));
                out = f32_to_bf16(s * uu);
            } else if (lt == 0) {
                atomicOr(p.status, kBadExpertId);
            }
            p.h[(size_t)q * I + row + lt] = out;
        }
        it += two ? 2 : 1;
    }
}

// ---------------------------------------------------------------- down -----
// CTA = a range of output rows (t, n) for every slot j; the warps of slot
// group j stream the down rows of expert ids[t][j]; the combine runs in
// shared memory after one barrier.  The first rows' weights are requested
// before the programmatic-launch wait (the routing is final by then: the
// gate/up kernel released this grid only after its own wait).

template <int TL, int KCH>
__global__ void __launch_bounds__(kDownThreads, 1)
down_decode_kernel(const DownParams p) {
    extern __shared__ __align__(16) float so[];  // [k][R]
    constexpr int TPW = 32 / TL;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lt = lane & (TL - 1);
    const unsigned mask = team_mask<TL>(lane);
    const int H = p.H, I = p.I, k = p.k, T = p.T;
    const int C = I >> 5;
    const size_t rc = (size_t)I >> 1, rs = (size_t)I >> 5;
    const int R = p.rows_per_cta;
    const int r0 = blockIdx.x * R;
    const int r1 = min(r0 + R, T * H);

    const int groups = kDownWarps / k;  // warps per slot
    const int j = warp % k, gi = warp / k;
    const int tps = groups * TPW;       // teams per slot
    const int ti = gi * TPW + lane / TL;
    const bool worker = gi < groups;

    // rows of this team: r0 + ti, r0 + ti + tps, ...; two per step
    int rr = r0 + ti;
    uint4 cw[2][KCH];
    uint32_t sc[2][KCH];
    bool bad[2] = {false, false};
    auto fetch = [&](int rbase) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = rbase + u * tps;
            const bool valid = worker && r < r1;
            const int t = valid ? r / H : 0;
            const int n = r - t * H;
            const int e = valid ? p.ids[t * k + j] : 0;
            bad[u] = valid && (e < 0 || e >= p.E);
            const bool ok = valid && !bad[u];
            const uint8_t *dc = nullptr, *ds = nullptr;
            if (ok) {
                dc = p.table[e].codes[2] + (size_t)n * rc;
                ds = p.table[e].scales[2] + (size_t)n * rs;
            }
            load_chunks<KCH>(dc, ds, ok, lt, C, cw[u], sc[u]);
        }
    };
    fetch(rr);

    pdl_wait();  // h comes from the gate/up kernel
    pdl_launch_dependents();

    uint32_t xw[KCH][16];
    int cur_tok = -1;
    float xs = 1.f;
    while (worker && rr < r1) {
        const int t = rr / H;
        if (t != cur_tok) {
            xs = pow2(stage_x<TL, KCH>(p.h + ((size_t)t * k + j) * I, lt, C, mask, xw));
            cur_tok = t;
        }
        // both rows of a step belong to token t unless the second crosses into
        // the next token; then it is recomputed in the next step
        const int rb = rr + tps;
        const bool second = rb < r1 && rb / H == t;
        float a0 = chunks_dot<KCH>(cw[0], sc[0], xw);
        float a1 = chunks_dot<KCH>(cw[1], sc[1], xw);
        a0 = team_add<TL>(a0, mask);
        a1 = team_add<TL>(a1, mask);
        const bool b0 = bad[0], b1 = bad[1];
        const int rnext = second ? rr + 2 * tps : rr + tps;
        if (rnext < r1) fetch(rnext);
        if (lt == 0) {
            so[j * R + (rr - r0)] = b0 ? 0.f : round_bf16(a0 * xs);
            if (b0) atomicOr(p.status, kBadExpertId);
            if (second) {
                so[j * R + (rb - r0)] = b1 ? 0.f : round_bf16(a1 * xs);
                if (b1) atomicOr(p.status, kBadExpertId);
            }
        }
        rr = rnext;
    }
    __syncthreads();

    // sequential BF16 combine in slot order, optional residual add
    for (int r = r0 + threadIdx.x; r < r1; r += kDownThreads) {
        const int t = r / H, n = r - t * H;
        float y = 0.f;
        for (int jj = 0; jj < k; ++jj) {
            const float o = so[jj * R + (r - r0)];
            const float wb = round_bf16(p.w[(size_t)t * k + jj]);
            y = round_bf16(y + round_bf16(o * wb));
            if (p.o_keep) p.o_keep[((size_t)t * k + jj) * H + n] = f32_to_bf16(o);
        }
        if (p.residual) y = round_bf16(bf16_to_f32(p.residual[r]) + y);
        p.y[r] = f32_to_bf16(y);
    }
}

// --------------------------------------------------------------- debug -----

__global__ void debug_dequant_kernel(const uint8_t *codes, const uint8_t *scales,
                                     long long groups, float *out) {
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= groups) return;
    const uint4 c = *reinterpret_cast<const uint4 *>(codes + g * 16);
    const float s = e8m0_to_f32(scales[g]);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t h[4];
        e2m1x8_to_f16x8(w[q], h);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            out[g * 32 + q * 8 + b * 2 + 0] = f16_bits_to_f32(h[b] & 0xFFFFu) * s;
            out[g * 32 + q * 8 + b * 2 + 1] = f16_bits_to_f32(h[b] >> 16) * s;
        }
    }
}

// -------------------------------------------------------------- launchers --

namespace {

template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t s, bool pdl, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// (TL, KCH) for K/32 = C chunks per row: a team of TL lanes, KCH chunks per lane.
void pick_team(int C, int &TL, int &KCH) {
    const int tls[4] = {32, 16, 8, 4};
    for (int i = 0; i < 4; ++i)
        if (C % tls[i] == 0 && C / tls[i] <= 4) {
            TL = tls[i];
            KCH = C / tls[i];
            return;
        }
    TL = 32;
    KCH = (C + 31) / 32;
}


template <int TL, int KCH>
cudaError_t launch_gu(const GateUpParams &p, int grid, cudaStream_t s, bool pdl) {
    return launch_ex(gateup_decode_kernel<TL, KCH>, dim3(grid), dim3(kGemvThreads), 0, s, pdl, p);
}

template <int TL, int KCH>
cudaError_t launch_dn(const DownParams &p, int grid, cudaStream_t s, bool pdl) {
    const size_t smem = down_decode_smem(p.T, p.k, p.I, p.rows_per_cta);
    if (smem > 48 * 1024) return cudaErrorInvalidValue;
    return launch_ex(down_decode_kernel<TL, KCH>, dim3(grid), dim3(kDownThreads), smem, s, pdl, p);
}

#define MOE_TEAM_DISPATCH(FN, C, ...)                                   \
    do {                                                                \
        int TL_, KCH_;                                                  \
        pick_team((C), TL_, KCH_);                                      \
        switch (TL_ * 10 + KCH_) {                                      \
        case 321: return FN<32, 1>(__VA_ARGS__);                        \
        case 322: return FN<32, 2>(__VA_ARGS__);                        \
        case 323: return FN<32, 3>(__VA_ARGS__);                        \
        case 324: return FN<32, 4>(__VA_ARGS__);                        \
        case 161: return FN<16, 1>(__VA_ARGS__);                        \
        case 162: return FN<16, 2>(__VA_ARGS__);                        \
        case 163: return FN<16, 3>(__VA_ARGS__);                        \
        case 164: return FN<16, 4>(__VA_ARGS__);                        \
        case 81: return FN<8, 1>(__VA_ARGS__);                          \
        case 82: return FN<8, 2>(__VA_ARGS__);                          \
        case 83: return FN<8, 3>(__VA_ARGS__);                          \
        case 84: return FN<8, 4>(__VA_ARGS__);                          \
        case 41: return FN<4, 1>(__VA_ARGS__);                          \
        case 42: return FN<4, 2>(__VA_ARGS__);                          \
        case 43: return FN<4, 3>(__VA_ARGS__);                          \
        case 44: return FN<4, 4>(__VA_ARGS__);                          \
        default: return cudaErrorInvalidValue;                          \
        }                                                               \
    } while (0)

}  // namespace

bool decode_shape_supported(int H, int I) {
    int tl, kch;
    pick_team(H / 32, tl, kch);
    if (kch > 4) return false;
    pick_team(I / 32, tl, kch);
    return kch <= 4;
}

size_t gateup_decode_smem(int, int) { return 0; }

size_t down_decode_smem(int, int k, int, int rows_per_cta) {
    return (size_t)k * rows_per_cta * 4;
}

cudaError_t launch_route(const RouteParams &p, cudaStream_t s, bool pdl) {
    const int tblocks = (p.T + kRouteWarps - 1) / kRouteWarps;
    return launch_ex(route_kernel, dim3(p.E, tblocks), dim3(kRouteThreads), 0, s, pdl, p);
}

cudaError_t launch_gateup_decode(const GateUpParams &p, int grid, cudaStream_t s, bool pdl) {
    MOE_TEAM_DISPATCH(launch_gu, p.H / 32, p, grid, s, pdl);
}

cudaError_t launch_down_decode(const DownParams &p, int grid, cudaStream_t s, bool pdl) {
    MOE_TEAM_DISPATCH(launch_dn, p.I / 32, p, grid, s, pdl);
}

cudaError_t launch_debug_dequant(const uint8_t *codes, const uint8_t *scales, int64_t n,
                                 float *out, cudaStream_t s) {
    const long long groups = n / 32;
    if (groups == 0) return cudaSuccess;
    const int bs = 256;
    const long long nb = (groups + bs - 1) / bs;
    debug_dequant_kernel<<<(unsigned)nb, bs, 0, s>>>(codes, scales, groups, out);
    return cudaGetLastError();
}

}  // namespace moe
