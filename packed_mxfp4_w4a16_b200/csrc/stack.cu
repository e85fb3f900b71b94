// stack.cu — the whole batch-1 decode step of a stack of MoE layers in one
// persistent launch.
//
// Sources (model card "LFM2.5-24B-A2B — Packed MXFP4 Inference"): "Grouped
// top-4 expert execution" (grouped gate and up GEMVs, SwiGLU, grouped down
// GEMV, fused combine with the sequential BF16 multiply/add rounding of a
// one-expert-at-a-time runner); "GPU routing inside resident-layer graphs"
// (router projection, bias, top-k and coefficients on the GPU, no id copy to
// the host); "Direct reads from GPU-resident weights" (experts read in place,
// no staging copy); "CUDA Graph lifetime and state management" (the RMS cells
// between MoE layers); table "Model and quantization" (E2M1 + E8M0 per 32,
// BF16 activations, FP32 accumulation, BF16 outputs).
//
// Why one launch.  At batch 1 a 24B-shaped layer streams 20 MB of packed
// weights (about 3 us of HBM time) but has three dependent grid-wide steps:
// the layer input must reach every CTA (each routes and multiplies the whole
// vector), the router logits must reach every CTA (each picks the experts whose
// rows it streams), and the SwiGLU vectors h must reach every CTA (each owns
// output rows of the down projection).  As separate kernels every step costs a
// grid drain and a launch; here the CTAs (one per SM, co-resident by a
// cooperative launch) stay in the kernel for all layers and hand each step over
// through 8-byte words {tag, value} in global memory, single-copy atomic, so a
// reader that sees this step's tag also sees the value written with it.  Every
// wait is bounded.
//
// One layer, CTA b of G:
//   A  the layer input r (the previous layer's tagged outputs, or the input
//      buffer for layer 0) into shared memory; weightless RMSNorm
//      xn = BF16(r / sqrt(mean(r^2) + 1e-6)); FP16 staging of xn for the GEMVs;
//      CTA b < E also computes router logit b (its router row was copied into
//      shared memory one layer ahead) and publishes it.
//   C  (producer warp) gathers all E logits, top-k + softmax, then requests
//      with bulk copies ALL of the CTA's weight bytes of the layer at once: its
//      share of the selected experts' gate/up rows (kStackChunks groups, one
//      mbarrier each, so the GEMVs start when the first group lands) and its
//      output rows of the down matrices (one mbarrier); and the router row of
//      the next layer.  The whole layer's ~20 MB is in flight from here on.
//   D  (23 consumer warps) one pair of gate/up rows per warp: E2M1 codes
//      decoded in registers against the FP16 activations, FP32 sums, SwiGLU,
//      the two h values published as one tagged word.
//   E  every CTA gathers all of h and stages it in shared memory as FP16.
//   F  the down GEMV of the CTA's output rows for every slot (rows already in
//      shared memory).
//   G  sequential BF16 combine in slot order and the residual add; the layer
//      output rows are published as tagged words (the next layer's input).
//
// The reduction orders are those of the one-launch-per-step kernels (router
// kernel, bulk-copy gate/up kernel, down kernel), so the results are
// bit-identical to running the layers one by one.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "down.cuh"

namespace moe {

namespace {

constexpr int kSWarps = kStackThreads / 32;   // 24
constexpr int kSProd = kSWarps - 1;           // producer warp
constexpr int kSCons = kSWarps - 1;           // gate/up consumer warps
constexpr int kSRouteWarps = kRouteThreads / 32;
constexpr size_t kStackSmemMax = 220 * 1024;  // dynamic; static shared memory is ~1.3 KB

static_assert(kStackThreads == kDownThreads, "the down phase uses the down kernel's team layout");

// Tag of step l of a launch: 26 bits of launch count, 6 bits of layer.
__device__ __forceinline__ unsigned stk_tag(unsigned base, int l) {
    return (base << 6) | (unsigned)l;
}

// Bounded poll of two adjacent tagged words (one 16-byte load of two
// single-copy-atomic 8-byte words) until both carry `tag`.  Gives up after
// `limit` polls, or early when the launch was aborted by another CTA.
__device__ __forceinline__ bool stk_poll2(const uint2 *p, unsigned tag, uint32_t &d0,
                                          uint32_t &d1, int limit, const unsigned *abort,
                                          unsigned base) {
    #pragma unroll 1
    for (int i = 0; i < limit; ++i) {
        uint2 a, c;
        ld_relaxed_gpu_2x64(p, a, c);
        if (a.x == tag && c.x == tag) {
            d0 = a.y;
            d1 = c.y;
            return true;
        }
        if ((i & 7) == 7 && ld_relaxed_gpu(abort) == base) return false;
        __nanosleep(32);
    }
    return false;
}

// By one warp: all n tagged logits (bounded), copied into s_logits.  Every
// lane returns the same verdict.  Out of line (once per layer).
static __device__ __noinline__ bool stk_gather_logits(const uint2 *ent, int n, unsigned tag,
                                                      float *s_logits, int limit,
                                                      const unsigned *abort, unsigned base) {
    const int lane = threadIdx.x & 31;
    unsigned seen = 0;  // entries j = lane + 32 s already copied (n <= 256)
    #pragma unroll 1
    for (int i = 0; i < limit; ++i) {
        bool all = true;
        #pragma unroll 1
        for (int j = lane, s = 0; j < n; j += 32, ++s) {
            if ((seen >> s) & 1u) continue;
            const uint2 v = ld_relaxed_gpu_v2(ent + j);
            if (v.x == tag) {
                s_logits[j] = __uint_as_float(v.y);
                seen |= 1u << s;
            } else {
                all = false;
            }
        }
        if (__all_sync(0xffffffffu, all)) {
            __syncwarp();
            return true;
        }
        if ((i & 7) == 7 && __any_sync(0xffffffffu, ld_relaxed_gpu(abort) == base)) return false;
        __nanosleep(32);
    }
    return false;
}

// By one warp: bulk copies of the CTA's gate/up rows of the selected experts.
// Copy group c covers the CTA's local row pairs [c ppc, (c+1) ppc); a group
// spans one or more slots q (segments), each giving four copies (gate codes,
// up codes, gate scales, up scales); the lane of (c, segment 0, matrix 0)
// announces the group's bytes on gbar[c].  Shared-memory layout: gate codes
// [NR][H/2], up codes [NR][H/2], gate scales [NR][H/32], up scales [NR][H/32].
static __device__ __noinline__ void stk_issue_gateup(const uint8_t *cb, const uint8_t *sb,
                                                     const ExpertPtrs *tab, size_t cstride,
                                                     size_t sstride, const int *s_ids, int E,
                                                     int H, int I, int pb0, int np, int ppc,
                                                     int nch, int NR, uint8_t *gu,
                                                     uint64_t *gbar) {
    const int lane = threadIdx.x & 31;
    const size_t rc = (size_t)H >> 1, rs = (size_t)H >> 5;
    const uint64_t pol = l2_evict_first_policy();  // rows are read once per token
    const int smax = (2 * ppc + I - 1) / I + 1;    // slots one group can touch
    const int ntask = nch * smax * 4;
    #pragma unroll 1
    for (int task = lane; task < ntask; task += 32) {
        const int c = task / (smax * 4), s = (task >> 2) % smax, m = task & 3;
        const int lp0 = c * ppc, lp1 = min(np, lp0 + ppc);
        const int g0 = 2 * (pb0 + lp0), g1 = 2 * (pb0 + lp1);  // global rows [g0, g1)
        const int qa = g0 / I, qb = (g1 - 1) / I;
        if (s == 0 && m == 0) {
            unsigned bytes = 0;
            #pragma unroll 1
            for (int q = qa; q <= qb; ++q) {
                const int e = s_ids[q];
                const int n = min(g1, (q + 1) * I) - max(g0, q * I);
                if (e >= 0 && e < E) bytes += (unsigned)(2 * n) * (unsigned)(rc + rs);
            }
            mbar_arrive_expect_tx(&gbar[c], bytes);
        }
        const int q = qa + s;
        if (q > qb) continue;
        const int e = s_ids[q];
        if (e < 0 || e >= E) continue;
        const int a = max(g0, q * I);
        const int n = min(g1, (q + 1) * I) - a;
        const size_t lr = (size_t)(a - 2 * pb0);  // local row
        const size_t i0 = (size_t)(a - q * I);    // row of the matrix
        const int mat = m & 1;                    // 0 gate, 1 up
        if (m < 2) {
            const uint8_t *src = cb ? cb + (size_t)(3 * e + mat) * cstride : tab[e].codes[mat];
            bulk_g2s_hint(gu + ((size_t)mat * NR + lr) * rc, src + i0 * rc, (unsigned)(n * rc),
                          &gbar[c], pol);
        } else {
            const uint8_t *src = cb ? sb + (size_t)(3 * e + mat) * sstride : tab[e].scales[mat];
            bulk_g2s_hint(gu + 2 * (size_t)NR * rc + ((size_t)mat * NR + lr) * rs, src + i0 * rs,
                          (unsigned)(n * rs), &gbar[c], pol);
        }
    }
}

// Router row e of a layer into shared memory (one bulk copy on *bar).
static __device__ __noinline__ void stk_issue_router(const uint16_t *wr, int e, int H,
                                                     uint16_t *dst, uint64_t *bar) {
    const uint64_t pol = l2_evict_last_policy();  // read again every token
    mbar_arrive_expect_tx(bar, (unsigned)H * 2u);
    bulk_g2s_hint(dst, wr + (size_t)e * H, (unsigned)H * 2u, bar, pol);
}

__device__ __forceinline__ float swiglu_h(float ag, float au, float xs) {
    const float g = round_bf16(ag * xs);
    const float u = round_bf16(au * xs);
    const float s = round_bf16(g / (1.0f + expf(-g)));
    return s * u;
}

}  // namespace

// KCH: 16-byte chunks per lane of a gate/up row (H = 32 * 32 * KCH at most);
// TLD / KCHD: the down phase's team of TLD lanes holding KCHD chunks each.
template <int KCH, int TLD, int KCHD>
__global__ void __launch_bounds__(kStackThreads, 1)
stack_decode_kernel(const __grid_constant__ StackParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    __shared__ __align__(8) uint64_t gbar[kStackChunks];
    __shared__ __align__(8) uint64_t dbar;
    __shared__ __align__(8) uint64_t rbar[2];
    __shared__ int s_ids[kMaxTopK];
    __shared__ float s_w[kMaxTopK];
    __shared__ float s_logits[kFusedMaxE];
    __shared__ float s_red[3][kSRouteWarps];
    __shared__ float s_xs[kMaxTopK];
    __shared__ unsigned s_hmax[kMaxTopK];
    __shared__ unsigned s_base;
    __shared__ int s_x16exp;
    __shared__ int s_fail;
    __shared__ int s_gu_armed, s_dn_armed;  // layer whose gate/up / down copies were issued
    __shared__ int s_rt_armed[2];           // layer whose router row went into buffer i

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = (int)blockIdx.x, G = (int)gridDim.x;
    const int E = p.E, H = p.H, I = p.I, k = p.k, L = p.L;
    const StackPlan &pl = p.plan;
    const int C = H >> 5;                                   // 32-element chunks per gate/up row
    const size_t rc = (size_t)H >> 1, rs = (size_t)H >> 5;  // gate/up row bytes: codes, scales
    const int nch8 = H >> 3;                                // 16-byte pieces of a BF16 vector
    const int limit = p.spin_limit;
    // this CTA's shares: gate/up row pairs [pb0, pb1), down rows [r0, r1)
    const int P = k * I / 2;
    const int pb0 = (int)((long long)P * b / G), pb1 = (int)((long long)P * (b + 1) / G);
    const int np = pb1 - pb0;
    const int NU = H / pl.U;
    const int r0 = pl.U * (int)((long long)NU * b / G);
    const int r1 = pl.U * (int)((long long)NU * (b + 1) / G);
    const int nch = (np + pl.ppc - 1) / pl.ppc;  // copy groups in use (same every layer)
    const int NR = 2 * pl.np_max;
    const int R = pl.R;
    uint8_t *gu = sm + pl.off_gu;
    uint8_t *rows_c = sm + pl.off_dn;                           // [k][R][I/2]
    uint8_t *rows_s = rows_c + (size_t)k * R * ((size_t)I >> 1);  // [k][R][I/32]
    uint16_t *rbuf = reinterpret_cast<uint16_t *>(sm + pl.off_rt);  // [2][H]
    uint32_t *sx = reinterpret_cast<uint32_t *>(sm + pl.off_sx);    // [H/2] layer input
    uint32_t *sx16 = reinterpret_cast<uint32_t *>(sm + pl.off_x16); // [H/2] FP16 routed vector
    uint32_t *sh = reinterpret_cast<uint32_t *>(sm + pl.off_sh);    // [k][I/2] FP16 h
    float *so = reinterpret_cast<float *>(sm + pl.off_so);          // [k][R] expert outputs

    if (tid == 0) {
        #pragma unroll 1
        for (int c = 0; c < kStackChunks; ++c) mbar_init(&gbar[c], 1);
        mbar_init(&dbar, 1);
        mbar_init(&rbar[0], 1);
        mbar_init(&rbar[1], 1);
        mbar_fence_init();
        // launches made so far by CTA b (every launch runs every CTA, so all
        // CTAs agree); written by the previous launch, complete before this one
        s_base = ld_relaxed_gpu(p.seq + b) + 1u;
        s_fail = 0;
        s_gu_armed = s_dn_armed = -1;
        s_rt_armed[0] = s_rt_armed[1] = -1;
    }
    __syncthreads();
    const unsigned base = s_base;
    if (warp == kSProd && lane == 0 && b < E) {
        stk_issue_router(p.layer[0].router_w, b, H, rbuf, &rbar[0]);
        s_rt_armed[0] = 0;
    }

    int l = 0;
    #pragma unroll 1
    for (; l < L; ++l) {
        const unsigned tag = stk_tag(base, l);
        const StackLayer &ly = p.layer[l];

        // ---- A: layer input r -> sx ----
        bool ok = true;
        if (l == 0) {
            const uint32_t *r32 = reinterpret_cast<const uint32_t *>(p.r);
            #pragma unroll 1
            for (int m = tid; m < (H >> 1); m += kStackThreads) sx[m] = r32[m];
        } else {
            #pragma unroll 1
            for (int m2 = tid; m2 < (H >> 2); m2 += kStackThreads) {
                uint32_t d0 = 0u, d1 = 0u;
                if (!stk_poll2(p.x_tag + 2 * m2, tag - 1u, d0, d1, limit, p.abort, base)) ok = false;
                sx[2 * m2] = d0;
                sx[2 * m2 + 1] = d1;
            }
            if (tid == 0 && ld_relaxed_gpu(p.abort) == base) ok = false;
        }
        if (!__syncthreads_and(ok)) break;
        if (b == 0 && p.r_hist) {
            uint32_t *dst = reinterpret_cast<uint32_t *>(p.r_hist + (size_t)l * H);
            #pragma unroll 1
            for (int m = tid; m < (H >> 1); m += kStackThreads) dst[m] = sx[m];
        }

        // ---- A: RMSNorm, router logit b, FP16 staging (threads of warps 0..7,
        // in the reduction order of the standalone router kernel) ----
        float acc = 0.f, amax = 0.f;
        if (tid < kRouteThreads) {
            uint4 xv[2];
            float ss = 0.f;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int c = tid + kRouteThreads * m;
                xv[m] = c < nch8 ? reinterpret_cast<const uint4 *>(sx)[c] : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t w4[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a = bf16_to_f32(w4[q] & 0xFFFFu), c2 = bf16_to_f32(w4[q] >> 16);
                    ss = fmaf(a, a, ss);
                    ss = fmaf(c2, c2, ss);
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) s_red[0][warp] = ss;
            asm volatile("bar.sync 1, %0;" ::"n"(kRouteThreads) : "memory");
            float tot = 0.f;
#pragma unroll
            for (int i = 0; i < kSRouteWarps; ++i) tot += s_red[0][i];
            const float inv = 1.0f / sqrtf(tot / (float)H + 1e-6f);
            uint4 wv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            const bool router = b < E;
            if (router) {
                // this layer's router row, copied one layer ahead
                if (!mbar_wait(&rbar[l & 1], (unsigned)(l >> 1) & 1u)) ok = false;
                const uint4 *wrow = reinterpret_cast<const uint4 *>(rbuf + (size_t)(l & 1) * H);
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int c = tid + kRouteThreads * m;
                    if (c < nch8) wv[m] = wrow[c];
                }
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int c = tid + kRouteThreads * m;
                if (c < nch8) {
                    uint32_t x4[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
                    const uint32_t r4[4] = {wv[m].x, wv[m].y, wv[m].z, wv[m].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        x4[q] = (uint32_t)f32_to_bf16(bf16_to_f32(x4[q] & 0xFFFFu) * inv) |
                                ((uint32_t)f32_to_bf16(bf16_to_f32(x4[q] >> 16) * inv) << 16);
                    xv[m] = make_uint4(x4[0], x4[1], x4[2], x4[3]);
                    if (b == 0 && p.xn_hist)
                        reinterpret_cast<uint4 *>(p.xn_hist + (size_t)l * H)[c] = xv[m];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float a = bf16_to_f32(x4[q] & 0xFFFFu), c2 = bf16_to_f32(x4[q] >> 16);
                        acc = fmaf(a, bf16_to_f32(r4[q] & 0xFFFFu), acc);
                        acc = fmaf(c2, bf16_to_f32(r4[q] >> 16), acc);
                        amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(c2)));
                    }
                }
            }
            acc = warp_sum(acc);
            amax = warp_max(amax);
            if (lane == 0) {
                s_red[1][warp] = acc;
                s_red[2][warp] = amax;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kRouteThreads) : "memory");
            if (router && tid == 0) {
                float logit = 0.f;
#pragma unroll
                for (int i = 0; i < kSRouteWarps; ++i) logit += s_red[1][i];
                if (ly.bias) logit += ly.bias[b];
                st_relaxed_gpu_v2(p.lg_tag + b, tag, __float_as_uint(logit));
                if (p.logits_hist) p.logits_hist[(size_t)l * E + b] = logit;
            }
            float mx = 0.f;
#pragma unroll
            for (int i = 0; i < kSRouteWarps; ++i) mx = fmaxf(mx, s_red[2][i]);
            const int c16 = f16_stage_exponent(mx);
            const float sf = pow2_neg(c16);
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int c = tid + kRouteThreads * m;
                if (c < nch8) {
                    const uint32_t x4[4] = {xv[m].x, xv[m].y, xv[m].z, xv[m].w};
                    uint4 o;
                    o.x = f32x2_to_f16x2(bf16_to_f32(x4[0] & 0xFFFFu) * sf, bf16_to_f32(x4[0] >> 16) * sf);
                    o.y = f32x2_to_f16x2(bf16_to_f32(x4[1] & 0xFFFFu) * sf, bf16_to_f32(x4[1] >> 16) * sf);
                    o.z = f32x2_to_f16x2(bf16_to_f32(x4[2] & 0xFFFFu) * sf, bf16_to_f32(x4[2] >> 16) * sf);
                    o.w = f32x2_to_f16x2(bf16_to_f32(x4[3] & 0xFFFFu) * sf, bf16_to_f32(x4[3] >> 16) * sf);
                    reinterpret_cast<uint4 *>(sx16)[c] = o;
                }
            }
            if (tid == 0) s_x16exp = c16;
        }
        if (!__syncthreads_and(ok)) break;

        // ---- C: routing and every copy of the layer (producer warp) ----
        if (warp == kSProd) {
            const bool got = stk_gather_logits(p.lg_tag, E, tag, s_logits, limit, p.abort, base);
            if (got) {
                int id;
                float w;
                warp_topk_any<true>(s_logits, E, k, lane, id, w);
                if (lane < k) {
                    s_ids[lane] = id;
                    s_w[lane] = w;
                    if (b == 0 && p.ids_hist) p.ids_hist[(size_t)l * k + lane] = id;
                    if (b == 0 && p.w_hist) p.w_hist[(size_t)l * k + lane] = w;
                }
                __syncwarp();
                stk_issue_gateup(ly.codes_base, ly.scales_base, ly.table, p.codes_stride,
                                 p.scales_stride, s_ids, E, H, I, pb0, np, pl.ppc, nch, NR, gu,
                                 gbar);
                __syncwarp();
                if (lane == 0) {
                    const DownSrc src = {ly.table, ly.codes_base, ly.scales_base, p.codes_stride,
                                         p.scales_stride};
                    issue_down_rows(src, E, H, I, k, s_ids, r0, r1, R, rows_c, rows_s, &dbar);
                    s_gu_armed = l;
                    s_dn_armed = l;
                } else if (lane == 1 && b < E && l + 1 < L) {
                    const int nb = (l + 1) & 1;
                    stk_issue_router(p.layer[l + 1].router_w, b, H, rbuf + (size_t)nb * H, &rbar[nb]);
                    s_rt_armed[nb] = l + 1;
                }
            } else if (lane == 0) {
                s_fail = 1;
            }
        }
        // consumers: this layer's activations while the routing is decided
        uint32_t xw[KCH][16];
#pragma unroll
        for (int u = 0; u < KCH; ++u) {
            const int c = lane + 32 * u;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 v = c < C ? reinterpret_cast<const uint4 *>(sx16)[c * 4 + q]
                                      : make_uint4(0u, 0u, 0u, 0u);
                xw[u][4 * q] = v.x;
                xw[u][4 * q + 1] = v.y;
                xw[u][4 * q + 2] = v.z;
                xw[u][4 * q + 3] = v.w;
            }
        }
        __syncthreads();
        if (s_fail) break;
        const float xs = pow2(s_x16exp);

        // ---- D: gate/up + SwiGLU, one row pair per consumer warp ----
        if (warp < kSCons) {
            #pragma unroll 1
            for (int pp = warp; pp < np; pp += kSCons) {
                if (!mbar_wait(&gbar[pp / pl.ppc], (unsigned)l & 1u)) {
                    ok = false;
                    break;
                }
                const int gr = 2 * (pb0 + pp);  // global row of the pair's first row
                const int q = gr / I;
                const int e = s_ids[q];
                const bool bad = e < 0 || e >= E;
                float v[4];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const size_t lr = (size_t)(2 * pp + rr);
                    uint4 cg[KCH], cu[KCH];
                    uint32_t sg[KCH], su[KCH];
#pragma unroll
                    for (int u = 0; u < KCH; ++u) {
                        const int c = lane + 32 * u;
                        if (c < C && !bad) {
                            cg[u] = *reinterpret_cast<const uint4 *>(gu + lr * rc + (size_t)c * 16);
                            cu[u] = *reinterpret_cast<const uint4 *>(gu + ((size_t)NR + lr) * rc +
                                                                     (size_t)c * 16);
                            sg[u] = gu[2 * (size_t)NR * rc + lr * rs + c];
                            su[u] = gu[2 * (size_t)NR * rc + ((size_t)NR + lr) * rs + c];
                        } else {
                            cg[u] = cu[u] = make_uint4(0u, 0u, 0u, 0u);
                            sg[u] = su[u] = 127u;
                        }
                    }
                    v[2 * rr] = chunks_dot<KCH>(cg, sg, xw);
                    v[2 * rr + 1] = chunks_dot<KCH>(cu, su, xw);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = warp_sum(v[i]);
                if (lane == 0) {
                    uint32_t word = 0u;
                    if (!bad) {
                        word = (uint32_t)f32_to_bf16(swiglu_h(v[0], v[1], xs)) |
                               ((uint32_t)f32_to_bf16(swiglu_h(v[2], v[3], xs)) << 16);
                    } else {
                        atomicOr(p.status, kBadExpertId);
                    }
                    st_relaxed_gpu_v2(p.h_tag + gr / 2, tag, word);
                }
            }
        }
        if (tid < k) s_hmax[tid] = 0u;
        if (!__syncthreads_and(ok)) break;

        // ---- E: all of h (tagged) -> FP16 in shared memory ----
        {
            const int npc = I >> 3;  // 8-element pieces per vector
            const int total = k * npc;
            uint4 *sv = reinterpret_cast<uint4 *>(sh);
            #pragma unroll 1
            for (int bs = warp * 32; bs < total; bs += kStackThreads) {
                const int i = bs + lane;
                const bool valid = i < total;
                float m = 0.f;
                int q = -1;
                if (valid) {
                    uint32_t d0 = 0u, d1 = 0u, d2 = 0u, d3 = 0u;
                    const uint2 *src = p.h_tag + (size_t)i * 4;
                    if (!stk_poll2(src, tag, d0, d1, limit, p.abort, base)) ok = false;
                    if (ok && !stk_poll2(src + 2, tag, d2, d3, limit, p.abort, base)) ok = false;
                    q = i / npc;
                    const int pi = i - q * npc;
                    sv[q * npc + h_piece(pi >> 2, pi & 3)] = make_uint4(d0, d1, d2, d3);
                    const uint32_t w4[4] = {d0, d1, d2, d3};
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        m = fmaxf(m, fmaxf(fabsf(bf16_to_f32(w4[r] & 0xFFFFu)),
                                           fabsf(bf16_to_f32(w4[r] >> 16))));
                }
                if (__all_sync(0xffffffffu, q == __shfl_sync(0xffffffffu, q, 0))) {
                    m = warp_max(m);
                    if (lane == 0 && q >= 0) atomicMax(s_hmax + q, __float_as_uint(m));
                } else if (valid) {
                    atomicMax(s_hmax + q, __float_as_uint(m));
                }
            }
            // the CTA's down rows (requested with the gate/up rows) must have landed
            if (tid == 0 && !mbar_wait(&dbar, (unsigned)l & 1u)) ok = false;
            if (!__syncthreads_and(ok)) break;
            #pragma unroll 1
            for (int i = tid; i < total; i += kStackThreads) {
                const float sf = pow2_neg(f16_stage_exponent(__uint_as_float(s_hmax[i / npc])));
                const uint4 v = sv[i];
                uint4 o;
                o.x = f32x2_to_f16x2(bf16_to_f32(v.x & 0xFFFFu) * sf, bf16_to_f32(v.x >> 16) * sf);
                o.y = f32x2_to_f16x2(bf16_to_f32(v.y & 0xFFFFu) * sf, bf16_to_f32(v.y >> 16) * sf);
                o.z = f32x2_to_f16x2(bf16_to_f32(v.z & 0xFFFFu) * sf, bf16_to_f32(v.z >> 16) * sf);
                o.w = f32x2_to_f16x2(bf16_to_f32(v.w & 0xFFFFu) * sf, bf16_to_f32(v.w >> 16) * sf);
                sv[i] = o;
            }
            if (tid < k) s_xs[tid] = pow2(f16_stage_exponent(__uint_as_float(s_hmax[tid])));
            __syncthreads();
        }

        // ---- F: down GEMV of the CTA's output rows, every slot ----
        {
            const DownSrc src = {ly.table, ly.codes_base, ly.scales_base, p.codes_stride,
                                 p.scales_stride};
            DownRows<TLD, KCHD, true> rows(H, I, k, E, R, r0, r1, src, s_ids, rows_c, rows_s);
            if (r0 < r1) {
                rows.fetch(rows.rr);
                rows.run(sh, s_xs, so, p.status);
            }
        }
        __syncthreads();

        // ---- G: sequential BF16 combine + residual; publish the layer output ----
        #pragma unroll 1
        for (int t = tid; 2 * t < r1 - r0; t += kStackThreads) {
            const int n = r0 + 2 * t;
            uint32_t word = 0u;
#pragma unroll
            for (int d = 0; d < 2; ++d) {
                float y = 0.f;
                for (int j = 0; j < k; ++j) {
                    const float o = so[j * R + (n + d - r0)];
                    const float wb = round_bf16(s_w[j]);
                    y = round_bf16(y + round_bf16(o * wb));
                }
                const uint32_t rb = (sx[(n + d) >> 1] >> (16 * ((n + d) & 1))) & 0xFFFFu;
                y = round_bf16(bf16_to_f32(rb) + y);
                word |= (uint32_t)f32_to_bf16(y) << (16 * d);
            }
            st_relaxed_gpu_v2(p.x_tag + n / 2, tag, word);
            if (l == L - 1) reinterpret_cast<uint32_t *>(p.r)[n / 2] = word;
        }
        __syncthreads();  // sx, so, s_w are rewritten by the next layer
    }

    if (l < L) {
        // gave up: record it, release the other CTAs, and let no copy of this
        // CTA outlive it (waits bounded; a wait already complete returns at once)
        if (tid == 0) {
            atomicOr(p.status, kTimeoutStatus);
            st_relaxed_gpu(p.abort, base);
            if (s_gu_armed == l) {
                for (int c = 0; c < nch; ++c) mbar_wait(&gbar[c], (unsigned)l & 1u);
            }
            if (s_dn_armed == l) mbar_wait(&dbar, (unsigned)l & 1u);
            for (int i = 0; i < 2; ++i)
                if (s_rt_armed[i] >= l) mbar_wait(&rbar[i], (unsigned)(s_rt_armed[i] >> 1) & 1u);
        }
    }
    if (tid == 0) st_relaxed_gpu(p.seq + b, base);
}

// ------------------------------------------------------------------ host --

namespace {

// (KCH, TLD, KCHD) variants built: gate/up rows up to H = 2048, the down
// teams of I in {384, 512, 1024, 1536, 2048}.
int stack_variant(int H, int I) {
    const int kch = (H / 32 + 31) / 32;
    int tl, kd;
    pick_team(I / 32, tl, kd);
    const int key = kch * 1000 + tl * 10 + kd;
    switch (key) {
    case 1043: return 0;
    case 1161: return 1;
    case 1321: return 2;
    case 2163: return 3;
    case 2322: return 4;
    case 2161: return 5;
    case 2321: return 6;
    default: return -1;
    }
}

template <int KCH, int TLD, int KCHD>
cudaError_t launch_stk(const StackParams &p, int grid, cudaStream_t s) {
    static PerDeviceOnce once;
    cudaError_t e = per_device_once(once, [] {
        return cudaFuncSetAttribute(stack_decode_kernel<KCH, TLD, KCHD>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kStackSmemMax);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kStackThreads);
    cfg.dynamicSmemBytes = p.plan.smem;
    cfg.stream = s;
    // cooperative: every CTA resident at once (they wait on one another), or
    // the launch fails
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, stack_decode_kernel<KCH, TLD, KCHD>, p);
}

size_t al128(size_t v) { return (v + 127) & ~(size_t)127; }

}  // namespace

bool stack_plan(int E, int H, int I, int k, int grid, StackPlan *pl) {
    if (grid < 1 || E < 1 || E > grid || E > kFusedMaxE || k < 1 || k > kMaxTopK || k > E)
        return false;
    if (H % 512 != 0 || H > 2048 || I % 128 != 0 || I > 4096) return false;
    if (stack_variant(H, I) < 0) return false;
    StackPlan s = {};
    s.U = (I % 256 == 0) ? 2 : 4;  // rows per unit: U * I/32 scale bytes are a 16-byte multiple
    const int P = k * I / 2;
    s.np_max = (P + grid - 1) / grid;
    s.ppc = (s.np_max + kStackChunks - 1) / kStackChunks;
    const int NU = H / s.U;
    s.R = s.U * ((NU + grid - 1) / grid);
    const size_t rc = (size_t)H / 2, rs = (size_t)H / 32;
    size_t off = 0;
    s.off_gu = (unsigned)off;
    off = al128(off + (size_t)2 * s.np_max * 2 * (rc + rs));
    s.off_dn = (unsigned)off;
    off = al128(off + (size_t)k * s.R * ((size_t)I / 2 + (size_t)I / 32));
    s.off_rt = (unsigned)off;
    off = al128(off + (size_t)2 * H * 2);
    s.off_sx = (unsigned)off;
    off = al128(off + (size_t)H * 2);
    s.off_x16 = (unsigned)off;
    off = al128(off + (size_t)H * 2);
    s.off_sh = (unsigned)off;
    off = al128(off + (size_t)k * I * 2);
    s.off_so = (unsigned)off;
    off = al128(off + (size_t)k * s.R * 4);
    s.smem = off;
    if (s.smem > kStackSmemMax) return false;
    *pl = s;
    return true;
}

cudaError_t launch_stack(const StackParams &p, int grid, cudaStream_t s) {
    switch (stack_variant(p.H, p.I)) {
    case 0: return launch_stk<1, 4, 3>(p, grid, s);
    case 1: return launch_stk<1, 16, 1>(p, grid, s);
    case 2: return launch_stk<1, 32, 1>(p, grid, s);
    case 3: return launch_stk<2, 16, 3>(p, grid, s);
    case 4: return launch_stk<2, 32, 2>(p, grid, s);
    case 5: return launch_stk<2, 16, 1>(p, grid, s);
    case 6: return launch_stk<2, 32, 1>(p, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
