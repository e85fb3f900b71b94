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

#include "down.cuh"

namespace moe {


// ------------------------------------------------------------------ route --
// route_logits_kernel: grid (E, ceil(T / kRouteTokensPerCta)); CTA (e, b)
// computes logit[t][e] for its tokens with all 256 threads on one dot product
// (each thread owns 16-byte chunks c = tid, tid + 256 of the row).  The
// router row is a constant input, fetched before the programmatic-launch
// wait.  With rmsnorm the CTA first reduces sum(r^2) of the token, rounds
// xn = BF16(r / sqrt(mean(r^2) + eps)) element-wise (CTA e = 0 also stores
// xn) and routes xn.  Top-k is done by the consumers of the logits.

constexpr int kRouteTokensPerCta = 8;
constexpr int kRouteMaxCpt = 2;  // 16-byte chunks per thread: H <= 2 * 256 * 8 = 4096

// Sum (or max) over the CTA with one barrier: warp partials to `red`
// (a buffer used only once per call site), every thread adds them up.
__device__ __forceinline__ float block_sum_route(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kRouteThreads / 32; ++i) s += red[i];
    return s;
}

__device__ __forceinline__ float block_max_route(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_max(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kRouteThreads / 32; ++i) s = fmaxf(s, red[i]);
    return s;
}

__global__ void __launch_bounds__(kRouteThreads)
route_logits_kernel(const RouteParams p) {
    __shared__ float red[3][kRouteThreads / 32];
    const int tid = threadIdx.x;
    const int e = blockIdx.x, H = p.H, E = p.E;
    const int nch = H >> 3;
    const uint16_t *row = p.wr + (size_t)e * H;
    const uint64_t pol = l2_evict_last_policy();  // reused by every token
    uint4 wv[kRouteMaxCpt];
#pragma unroll
    for (int m = 0; m < kRouteMaxCpt; ++m) {
        const int c = tid + kRouteThreads * m;
        wv[m] = c < nch ? ld_hint16(row + (size_t)c * 8, pol) : make_uint4(0u, 0u, 0u, 0u);
    }
    pdl_wait();
    pdl_launch_dependents();

    const int t0 = blockIdx.y * kRouteTokensPerCta;
    const int t1 = min(p.T, t0 + kRouteTokensPerCta);
    #pragma unroll 1
    for (int t = t0; t < t1; ++t) {
        if (t > t0) __syncthreads();  // red[] is reused for the next token
        const uint16_t *xt = p.x + (size_t)t * H;
        uint4 xv[kRouteMaxCpt];
        float ss = 0.f;
#pragma unroll
        for (int m = 0; m < kRouteMaxCpt; ++m) {
            const int c = tid + kRouteThreads * m;
            xv[m] = c < nch ? *reinterpret_cast<const uint4 *>(xt + (size_t)c * 8)
                            : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w4[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float a = bf16_to_f32(w4[q] & 0xFFFFu), b = bf16_to_f32(w4[q] >> 16);
                ss = fmaf(a, a, ss);
                ss = fmaf(b, b, ss);
            }
        }
        float inv = 1.f;
        if (p.rmsnorm) inv = 1.0f / sqrtf(block_sum_route(ss, red[0]) / (float)H + p.eps);
        float acc = 0.f, amax = 0.f;
#pragma unroll
        for (int m = 0; m < kRouteMaxCpt; ++m) {
            const int c = tid + kRouteThreads * m;
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
                xv[m] = make_uint4(x4[0], x4[1], x4[2], x4[3]);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a = bf16_to_f32(x4[q] & 0xFFFFu), b = bf16_to_f32(x4[q] >> 16);
                    acc = fmaf(a, bf16_to_f32(r4[q] & 0xFFFFu), acc);
                    acc = fmaf(b, bf16_to_f32(r4[q] >> 16), acc);
                    amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
                }
            }
        }
        const float logit = block_sum_route(acc, red[1]);
        if (tid == 0) {
            // sigmoid scoring keeps the logit unbiased (the bias enters the
            // selection key in the top-k)
            const float v = (p.bias && !p.sigmoid) ? logit + p.bias[e] : logit;
            p.logits_ws[(size_t)t * E + e] = v;
            if (p.logits_out) p.logits_out[(size_t)t * E + e] = v;
        }
        if (e == 0 && p.x16) {
            // the expert GEMVs' FP16 staging of the routed vector, done once here
            const int c16 = f16_stage_exponent(block_max_route(amax, red[2]));
            const float sf = pow2_neg(c16);
#pragma unroll
            for (int m = 0; m < kRouteMaxCpt; ++m) {
                const int c = tid + kRouteThreads * m;
                if (c < nch) {
                    const uint32_t x4[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
                    uint4 o;
                    o.x = f32x2_to_f16x2(bf16_to_f32(x4[0] & 0xFFFFu) * sf, bf16_to_f32(x4[0] >> 16) * sf);
                    o.y = f32x2_to_f16x2(bf16_to_f32(x4[1] & 0xFFFFu) * sf, bf16_to_f32(x4[1] >> 16) * sf);
                    o.z = f32x2_to_f16x2(bf16_to_f32(x4[2] & 0xFFFFu) * sf, bf16_to_f32(x4[2] >> 16) * sf);
                    o.w = f32x2_to_f16x2(bf16_to_f32(x4[3] & 0xFFFFu) * sf, bf16_to_f32(x4[3] >> 16) * sf);
                    *reinterpret_cast<uint4 *>(p.x16 + (size_t)t * (H >> 1) + (size_t)c * 4) = o;
                }
            }
            if (tid == 0) p.x16_exp[t] = c16;
        }
    }
}

// topk_kernel: grid ceil(T / 8), 256 threads; warp w selects for token
// 8 * blockIdx.x + w and writes ids / w (standalone routing call).
__global__ void __launch_bounds__(kRouteThreads)
topk_kernel(const RouteParams p) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (kRouteThreads / 32) + (threadIdx.x >> 5);
    if (t >= p.T) return;
    int id;
    float w;
    if (p.sigmoid)
        warp_topk_any<false, true>(p.logits_ws + (size_t)t * p.E, p.E, p.k, lane, id, w, p.bias);
    else
        warp_topk_any(p.logits_ws + (size_t)t * p.E, p.E, p.k, lane, id, w);
    if (lane < p.k) {
        p.ids[(size_t)t * p.k + lane] = id;
        p.w[(size_t)t * p.k + lane] = w;
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

    __shared__ int s_ids[kDecodeMaxT * kMaxTopK];
    pdl_wait();  // x and the routing come from earlier kernels
    pdl_launch_dependents();
    if (p.ids) {
        for (int q = threadIdx.x; q < p.T * k; q += kGemvThreads) s_ids[q] = p.ids[q];
    } else {
        route_into_smem(p.logits, p.T, p.E, k, s_ids, nullptr, p.ids_out, p.w_out);
    }
    __syncthreads();
    if (p.prefetch_down && warp == kGemvWarps - 1) prefetch_down_slice(p, s_ids, lane);

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

    #pragma unroll 1
    while (it < end) {
        const int q = (int)(it / I);
        const int row = (int)(it - (long long)q * I);
        // a second row of the same pair in this step if there is one
        const bool two = (it + 1 < end) && (row + 1 < I);
        if (q != cur_q) {
            const int e = s_ids[q];
            bad = (e < 0 || e >= p.E);
            if (!bad && p.codes_base) {
                gc = p.codes_base + (size_t)(3 * e) * p.codes_stride;
                uc = p.codes_base + (size_t)(3 * e + 1) * p.codes_stride;
                gs = p.scales_base + (size_t)(3 * e) * p.scales_stride;
                us = p.scales_base + (size_t)(3 * e + 1) * p.scales_stride;
            } else if (!bad) {
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
            load_chunks<TL, KCH>(gc + r * rc, gs + r * rs, ok, lt, C, cg[u], sg[u]);
            load_chunks<TL, KCH>(uc + r * rc, us + r * rs, ok, lt, C, cu[u], su[u]);
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

// ------------------------------------------------- gate / up, bulk copies --
// Rows of the selected experts stream into a shared-memory ring with bulk
// copies (ring_produce / ring_consume).  For T = 1 the whole CTA range (~40
// rows, ~90 KB) is requested at once, so the DRAM sees the layer's entire
// gate/up stream immediately.

template <int KCH, bool NV>
__global__ void __launch_bounds__(kTmaThreads, 1)
gateup_tma_kernel(const GateUpParams p) {
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t full[kTmaMaxSlots];
    __shared__ __align__(8) uint64_t empty[kTmaMaxSlots];
    __shared__ int s_ids[kDecodeMaxT * kMaxTopK];
    __shared__ ExpertPtrs s_tab[kDecodeMaxT * kMaxTopK];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = p.H, k = p.k, T = p.T, E = p.E;
    const int C = H >> 5;
    const RingGeom g = ring_geom(p);
    if (threadIdx.x == 0) ring_init(g, full, empty);
    __syncthreads();
    pdl_wait();  // x and the routing come from earlier kernels
    pdl_launch_dependents();

    if (warp == kTmaConsumers) {
        // ---- producer warp: the call's routing, then the ring ----
        const int P = T * k;
        if (p.ids) {
            #pragma unroll 1
            for (int q = lane; q < P; q += 32) s_ids[q] = p.ids[q];
        } else {
            #pragma unroll 1
            for (int t = 0; t < T; ++t)
                topk_token_to_smem(p.logits + (size_t)t * E, E, k, s_ids + t * k,
                                   blockIdx.x == 0 ? p.ids_out + (p.ids_out ? t * k : 0) : nullptr,
                                   blockIdx.x == 0 ? p.w_out + (p.w_out ? t * k : 0) : nullptr);
        }
        __syncwarp();
        ring_produce(p, g, ring, full, empty, s_ids, s_tab, lane, [] {});
        return;
    }

    // ---- consumer warps ----
    // FP16 activations of token `tok` into registers: loaded as staged by the
    // router when available, else staged here.  Plain (L1-allocating) loads:
    // every warp of the CTA reads the same vector, so one L2 read per SM
    // serves all of them.
    ring_consume<KCH, NV>(p, g, ring, full, empty, s_ids, warp, lane,
                      [&](int tok, uint32_t (&xw)[KCH][16]) -> float {
        if (p.x16) {
            const uint32_t *xv = p.x16 + (size_t)tok * (H >> 1);
#pragma unroll
            for (int u = 0; u < KCH; ++u) {
                const int c = lane + 32 * u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = c < C ? reinterpret_cast<const uint4 *>(xv + (size_t)c * 16)[q]
                                          : make_uint4(0u, 0u, 0u, 0u);
                    xw[u][4 * q] = v.x;
                    xw[u][4 * q + 1] = v.y;
                    xw[u][4 * q + 2] = v.z;
                    xw[u][4 * q + 3] = v.w;
                }
            }
            return pow2(p.x16_exp[tok]);
        }
        return pow2(stage_x<32, KCH>(p.x + (size_t)tok * H, lane, C, 0xffffffffu, xw));
    }, [&](size_t idx, uint16_t v) { p.h[idx] = v; });
}

// ---------------------------------------------------------------- down -----
// CTA = a range of output rows (t, n) for every slot j.  Before the
// programmatic-launch wait (the routing is final by then: the gate/up grid
// released this one only after its own wait) the CTA selects the experts and
// requests its first down rows.  After the wait it stages the k*T SwiGLU
// vectors h once into shared memory as FP16, then teams of TL lanes (slot
// group j = warp % k) stream their rows against them.  Expert outputs meet in
// shared memory for the sequential BF16 combine.

// Routing handed over by CTA blockIdx.x of the fused router + gate/up kernel
// of the same call (RouteHandoff), by one warp: lane q < P polls (bounded) its
// two tagged entries until both carry the expected tag; lane 0 acknowledges.
// A timeout flags the status, marks the slots invalid (id -1: zero output)
// and resynchronises the acknowledgement.  Out of line.
static __device__ __noinline__ void take_handoff(const RouteHandoff h, int P, int *s_ids,
                                                 float *s_w, unsigned *status) {
    const int lane = threadIdx.x & 31;
    const int slot = (int)blockIdx.x;
    const unsigned want = ld_relaxed_gpu(h.ack + slot) + 1u;
    bool ok = true;
    if (lane < P) {
        const uint2 *e = h.ent + ((size_t)slot * kHandStride + lane) * 2;
        uint2 a = make_uint2(0u, 0u), b = make_uint2(0u, 0u);
        ok = false;
        #pragma unroll 1
        for (int i = 0; i < kMaxSpin && !ok; ++i) {
            a = ld_relaxed_gpu_v2(e);
            b = ld_relaxed_gpu_v2(e + 1);
            ok = a.x == want && b.x == want;
        }
        s_ids[lane] = ok ? (int)a.y : -1;
        s_w[lane] = ok ? __uint_as_float(b.y) : 0.f;
    }
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (lane == 0) {
        if (!all_ok) atomicOr(status, kTimeoutStatus);
        st_relaxed_gpu(h.ack + slot, all_ok ? want : ld_relaxed_gpu(h.seq + slot));
    }
}

// SR: every down row of the CTA is copied into shared memory with bulk copies
// before the programmatic-launch wait (rows: [k][R] codes, then [k][R] scales);
// otherwise each team streams its rows from global memory two at a time.
template <int TL, int KCH, bool SR, bool NV>
__global__ void __launch_bounds__(kDownThreads, 1)
down_decode_kernel(const DownParams p) {
    extern __shared__ __align__(16) uint8_t sm[];
    const int warp = threadIdx.x >> 5;
    const int H = p.H, I = p.I, k = p.k, T = p.T;
    const int R = p.rows_per_cta;
    const int r0 = blockIdx.x * R;
    const int r1 = min(r0 + R, T * H);
    const int P = T * k;
    uint32_t *sh = reinterpret_cast<uint32_t *>(sm);                       // [P][I/2] FP16 words
    float *so = reinterpret_cast<float *>(sm + (size_t)P * I * 2);         // [k][R]
    uint8_t *rows_c = sm + down_rows_offset(T, k, I, R);                   // SR: [k][R][I/2]
    uint8_t *rows_s = rows_c + (size_t)k * R * ((size_t)I >> 1);           // SR: [k][R][I/32 or /16]
    __shared__ __align__(8) uint64_t s_rbar;
    __shared__ int s_ids[kDecodeMaxT * kMaxTopK];
    __shared__ float s_w[kDecodeMaxT * kMaxTopK];
    __shared__ float s_xs[kDecodeMaxT * kMaxTopK];
    __shared__ float s_gs[kDecodeMaxT * kMaxTopK];  // NV: each pair's down multiplier
    __shared__ unsigned s_hmax[kDecodeMaxT * kMaxTopK];

    // routing for this call's tokens
    if (threadIdx.x < P) s_hmax[threadIdx.x] = 0u;
    if (SR && threadIdx.x == 0) {
        mbar_init(&s_rbar, 1);
        mbar_fence_init();
    }
    if (p.ids) {
        for (int q = threadIdx.x; q < P; q += kDownThreads) {
            s_ids[q] = __ldcg(p.ids + q);
            s_w[q] = __ldcg(p.w + q);
        }
    } else if (p.logits) {
        route_into_smem(p.logits, T, p.E, k, s_ids, s_w, nullptr, nullptr);
    } else if (warp == 0) {
        take_handoff(p.hand, P, s_ids, s_w, p.status);
    }
    __syncthreads();

    const DownSrc src = {p.table, p.codes_base, p.scales_base, p.codes_stride, p.scales_stride};
    if (NV && threadIdx.x < P) {  // read before the barriers inside stage_h_block
        const int e = s_ids[threadIdx.x];
        s_gs[threadIdx.x] = (e >= 0 && e < p.E) ? __ldg(p.gscale + 2 * e + 1) : 0.f;
    }
    DownRows<TL, KCH, SR, NV> rows(H, I, k, p.E, R, r0, r1, src, s_ids, rows_c, rows_s);
    if (SR) {
        if (threadIdx.x == 0)
            issue_down_rows(src, p.E, H, I, k, s_ids, r0, r1, R, rows_c, rows_s, &s_rbar,
                            NV ? 1 : 0);
    } else {
        rows.fetch(rows.rr);
    }

    pdl_wait();  // h comes from the gate/up kernel
    pdl_launch_dependents();

    // stage every h[t][j] once into shared memory as FP16
    stage_h_block(p.h, P, I, sh, s_xs, s_hmax);
    bool rows_ok = true;
    if (SR) {
        rows_ok = __syncthreads_and(mbar_wait(&s_rbar, 0u)) != 0;  // uniform over the CTA
        if (!rows_ok && threadIdx.x == 0) atomicOr(p.status, kTimeoutStatus);
    }
    if (rows_ok) rows.run(sh, s_xs, so, p.status, s_gs);
    __syncthreads();

    // sequential BF16 combine in slot order, optional residual add
    down_combine(r0, r1, H, k, R, so, s_w, p.residual, p.y, p.o_keep);
    // no row copy may outlive the CTA (complete unless its wait timed out)
    if (SR && !rows_ok && threadIdx.x == 0) mbar_wait(&s_rbar, 0u);
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

template <int TL, int KCH>
cudaError_t launch_gu(const GateUpParams &p, int grid, cudaStream_t s, bool pdl) {
    return launch_ex(gateup_decode_kernel<TL, KCH>, dim3(grid), dim3(kGemvThreads), 0, s, pdl, p);
}

template <int TL, int KCH, bool SR, bool NV>
cudaError_t launch_dn_v(const DownParams &p, int grid, size_t smem, cudaStream_t s, bool pdl) {
    // once per device (the attribute belongs to the current device's context)
    static PerDeviceOnce once;
    const cudaError_t attr = per_device_once(once, [] {
        return cudaFuncSetAttribute(down_decode_kernel<TL, KCH, SR, NV>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDownSmemMax);
    });
    if (attr != cudaSuccess) return attr;
    return launch_ex(down_decode_kernel<TL, KCH, SR, NV>, dim3(grid), dim3(kDownThreads), smem, s,
                     pdl, p);
}

// The shared-memory-rows variant when its copies are 16-byte shaped (I a
// multiple of 512) and the rows fit; else rows stream from global memory.
template <int TL, int KCH, bool NV>
cudaError_t launch_dn(const DownParams &p, int grid, cudaStream_t s, bool pdl) {
    const size_t smem = down_decode_smem(p.T, p.k, p.I, p.rows_per_cta);
    if (smem > kDownSmemMax) return cudaErrorInvalidValue;
    const size_t smem_sr = down_rows_smem(p.T, p.k, p.I, p.rows_per_cta, NV ? 1 : 0);
    if (p.I % 512 == 0 && smem_sr <= kDownSmemMax)
        return launch_dn_v<TL, KCH, true, NV>(p, grid, smem_sr, s, pdl);
    return launch_dn_v<TL, KCH, false, NV>(p, grid, smem, s, pdl);
}
template <int TL, int KCH>
cudaError_t launch_dn_mx(const DownParams &p, int grid, cudaStream_t s, bool pdl) {
    return launch_dn<TL, KCH, false>(p, grid, s, pdl);
}
template <int TL, int KCH>
cudaError_t launch_dn_nv(const DownParams &p, int grid, cudaStream_t s, bool pdl) {
    return launch_dn<TL, KCH, true>(p, grid, s, pdl);
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

bool gateup_tma_supported(int H) { return H % 512 == 0 && H <= 4096; }

int gateup_tma_slots(int H, int nv) {
    const size_t sb = tma_slot_bytes(H, nv);
    size_t n = kTmaSmemBudget / sb;
    if (n > (size_t)kTmaMaxSlots) n = kTmaMaxSlots;
    return (int)n;
}

template <int KCH, bool NV>
cudaError_t launch_gu_tma(const GateUpParams &p, int grid, cudaStream_t s, bool pdl) {
    const size_t smem = (size_t)p.nslots * tma_slot_bytes(p.H, NV ? 1 : 0);
    if (smem > kTmaSmemBudget) return cudaErrorInvalidValue;
    // once per device (the attribute belongs to the current device's context)
    static PerDeviceOnce once;
    const cudaError_t attr = per_device_once(once, [] {
        return cudaFuncSetAttribute(gateup_tma_kernel<KCH, NV>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kTmaSmemBudget);
    });
    if (attr != cudaSuccess) return attr;
    return launch_ex(gateup_tma_kernel<KCH, NV>, dim3(grid), dim3(kTmaThreads), smem, s, pdl, p);
}

bool decode_shape_supported(int H, int I) {
    int tl, kch;
    pick_team(H / 32, tl, kch);
    if (kch > 4) return false;
    pick_team(I / 32, tl, kch);
    return kch <= 4;
}

size_t gateup_decode_smem(int, int) { return 0; }

size_t down_decode_smem(int T, int k, int I, int rows_per_cta) {
    return (size_t)T * k * I * 2 + (size_t)k * rows_per_cta * 4;
}

cudaError_t launch_route_logits(const RouteParams &p, cudaStream_t s, bool pdl) {
    const int tblocks = (p.T + kRouteTokensPerCta - 1) / kRouteTokensPerCta;
    return launch_ex(route_logits_kernel, dim3(p.E, tblocks), dim3(kRouteThreads), 0, s, pdl, p);
}

cudaError_t launch_topk(const RouteParams &p, cudaStream_t s, bool pdl) {
    const int blocks = (p.T + kRouteThreads / 32 - 1) / (kRouteThreads / 32);
    return launch_ex(topk_kernel, dim3(blocks), dim3(kRouteThreads), 0, s, pdl, p);
}

cudaError_t launch_route(const RouteParams &p, cudaStream_t s, bool pdl) {
    cudaError_t e = launch_route_logits(p, s, pdl);
    if (e != cudaSuccess) return e;
    return launch_topk(p, s, pdl);
}

cudaError_t launch_gateup_decode(const GateUpParams &p, int grid, cudaStream_t s, bool pdl) {
    if (p.nslots >= 2 && gateup_tma_supported(p.H)) {
        switch ((p.H / 32 + 31) / 32 + (p.nv ? 4 : 0)) {
        case 1: return launch_gu_tma<1, false>(p, grid, s, pdl);
        case 2: return launch_gu_tma<2, false>(p, grid, s, pdl);
        case 3: return launch_gu_tma<3, false>(p, grid, s, pdl);
        case 4: return launch_gu_tma<4, false>(p, grid, s, pdl);
        case 5: return launch_gu_tma<1, true>(p, grid, s, pdl);
        case 6: return launch_gu_tma<2, true>(p, grid, s, pdl);
        case 7: return launch_gu_tma<3, true>(p, grid, s, pdl);
        case 8: return launch_gu_tma<4, true>(p, grid, s, pdl);
        default: return cudaErrorInvalidValue;
        }
    }
    if (p.nv) return cudaErrorInvalidValue;  // NVFP4 runs on the bulk-copy kernel only
    MOE_TEAM_DISPATCH(launch_gu, p.H / 32, p, grid, s, pdl);
}

cudaError_t launch_down_decode(const DownParams &p, int grid, cudaStream_t s, bool pdl) {
    if (p.nv) {
        MOE_TEAM_DISPATCH(launch_dn_nv, p.I / 32, p, grid, s, pdl);
    } else {
        MOE_TEAM_DISPATCH(launch_dn_mx, p.I / 32, p, grid, s, pdl);
    }
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
