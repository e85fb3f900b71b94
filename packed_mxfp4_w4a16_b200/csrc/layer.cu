// layer.cu — router and gate/up of a decode layer (T <= 4 tokens) in one
// launch.
//
// Sources (model card "LFM2.5-24B-A2B — Packed MXFP4 Inference"): "GPU routing
// inside resident-layer graphs" (router projection, bias, top-k and the
// routing coefficients computed on the GPU, no id copy to the host) and
// "Grouped top-4 expert execution" (grouped gate and up GEMVs + SwiGLU);
// table "Model and quantization" (BF16 router and activations, FP32
// accumulation).
//
// One CTA per SM (grid = SM count, all resident together).  CTA b owns the router
// rows of experts b, b + G, ...; it fetches its first row into registers before
// the programmatic-launch wait (a constant input).  After the wait every CTA
// loads the layer input and applies the weightless RMSNorm (when asked) into
// shared memory; CTA b computes its experts' logits and publishes each as one
// 8-byte word {tag, logit} in the workspace.  The producer warp of every CTA
// polls the E words of each token (bounded) until they carry this call's tag,
// selects the experts (top-k + softmax) and streams the CTA's gate/up rows
// through the shared-memory ring exactly as the unfused gate/up kernel does;
// the consumer warps read the routed vector from shared memory.
//
// Tags: workspace counter seq[b] counts the fused calls made on this
// workspace; every call runs all G CTAs, so seq[b] is the same for every b and
// tag = seq[b] + 1 is unique to the call.  The routing goes to the down kernel
// of the same call through the per-CTA handoff, with the same tag.
//
// With a down team shape (TLD > 0) the same grid also runs the down GEMV and
// the combine: the producer issues bulk copies of the CTA's down rows into
// shared memory right after routing; the consumers write each h value with
// this call's tag as one 8-byte word; every CTA then stages all of h, each
// piece re-read (bounded) until it carries the tag, and reduces its rows as
// the standalone down kernel does.  No kernel boundary and no grid-wide wait
// remain inside the layer: each CTA waits only for the h values it reads.
//
// Every reduction follows the standalone router kernel's order (its thread
// tid owns the 16-byte pieces tid and tid + 256 of a row; warp sums; the 8
// warp partials added in order), so x_norm, the logits and the routing are
// bit-identical to the unfused path.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "down.cuh"

namespace moe {

namespace {

constexpr int kRouteWarps = kRouteThreads / 32;
constexpr size_t kFusedSmemBudget = 216 * 1024;  // dynamic shared memory of the fused kernel

// acc += the 8 BF16 products of two 16-byte pieces, in element order, each a
// fused multiply-add of the exact BF16 x BF16 product into FP32.
__device__ __forceinline__ float dot8_bf16(const uint4 x, const uint4 w, float acc) {
    asm("{ .reg .b16 x0, x1, w0, w1;\n"
        "mov.b32 {x0, x1}, %1; mov.b32 {w0, w1}, %5;\n"
        "fma.rn.f32.bf16 %0, x0, w0, %0; fma.rn.f32.bf16 %0, x1, w1, %0;\n"
        "mov.b32 {x0, x1}, %2; mov.b32 {w0, w1}, %6;\n"
        "fma.rn.f32.bf16 %0, x0, w0, %0; fma.rn.f32.bf16 %0, x1, w1, %0;\n"
        "mov.b32 {x0, x1}, %3; mov.b32 {w0, w1}, %7;\n"
        "fma.rn.f32.bf16 %0, x0, w0, %0; fma.rn.f32.bf16 %0, x1, w1, %0;\n"
        "mov.b32 {x0, x1}, %4; mov.b32 {w0, w1}, %8;\n"
        "fma.rn.f32.bf16 %0, x0, w0, %0; fma.rn.f32.bf16 %0, x1, w1, %0; }"
        : "+f"(acc)
        : "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w));
    return acc;
}

// By one warp: wait (bounded) until the n tagged logit words carry `tag`,
// copying the values into s_logits.  Returns false on timeout.  Out of line.
static __device__ __noinline__ bool gather_logits(const uint2 *ent, int n, unsigned tag,
                                                  float *s_logits) {
    const int lane = threadIdx.x & 31;
    bool ok = false;
    #pragma unroll 1
    for (int i = 0; i < kMaxSpin && !ok; ++i) {
        bool mine = true;
        #pragma unroll 2
        for (int j = lane; j < n; j += 32) {
            const uint2 v = ld_relaxed_gpu_v2(ent + j);
            if (v.x == tag)
                s_logits[j] = __uint_as_float(v.y);
            else
                mine = false;
        }
        ok = __all_sync(0xffffffffu, mine);
        if (!ok) __nanosleep(128);  // fewer polls on lines other CTAs are writing
    }
    return ok;
}

// Top-k + softmax of every token from the logits in shared memory, by the
// calling warp, into s_ids / s_w ([T][k]).  Out of line: it runs once per call.
static __device__ __noinline__ void fused_topk(const float *s_logits, int T, int E, int k,
                                               int *s_ids, float *s_w) {
    const int lane = threadIdx.x & 31;
    #pragma unroll 1
    for (int t = 0; t < T; ++t) {
        int id;
        float w;
        warp_topk_any<true>(s_logits + t * E, E, k, lane, id, w);
        if (lane < k) {
            s_ids[t * k + lane] = id;
            s_w[t * k + lane] = w;
        }
    }
}

}  // namespace

// TLD == 0: router + gate/up (a down kernel follows); TLD > 0: the whole
// layer, down teams of TLD lanes holding KCHD chunks each.
template <int KCH, int TLD, int KCHD>
__global__ void __launch_bounds__(kTmaThreads, 1)
layer_kernel(const GateUpParams p, const FusedRouteParams r, const LayerDownParams dp) {
    static_assert(kTmaThreads == kDownThreads, "one CTA shape for both phases");
    constexpr bool kWhole = TLD > 0;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t full[kTmaMaxSlots];
    __shared__ __align__(8) uint64_t empty[kTmaMaxSlots];
    __shared__ int s_ids[kDecodeMaxT * kMaxTopK];
    __shared__ float s_w[kDecodeMaxT * kMaxTopK];
    __shared__ ExpertPtrs s_tab[kDecodeMaxT * kMaxTopK];
    __shared__ float s_logits[kDecodeMaxT * kFusedMaxE];
    __shared__ float s_red[kRouteWarps][kDecodeMaxT][2];
    __shared__ int s_xexp[kDecodeMaxT];
    __shared__ unsigned s_tag;
    __shared__ __align__(8) uint64_t s_dbar;               // kWhole: the CTA's down rows
    __shared__ float s_xs[kDecodeMaxT * kMaxTopK];          // kWhole: h staging scales
    __shared__ unsigned s_hmax[kDecodeMaxT * kMaxTopK];     // kWhole: h staging maxima
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int H = p.H, k = p.k, T = p.T, E = p.E;
    const int C = H >> 5;
    const int nch = H >> 3;  // 16-byte pieces of one BF16 vector
    const int G = (int)gridDim.x;
    uint16_t *sx = reinterpret_cast<uint16_t *>(ring + r.region_bytes);  // [T][H] routed vector
    const bool rthread = threadIdx.x < kRouteThreads;
    const RingGeom g = ring_geom(p);

    // the first router row of this CTA (a constant input), while the previous
    // kernel drains
    uint4 wv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    if (rthread && (int)blockIdx.x < E) {
        const uint4 *row = reinterpret_cast<const uint4 *>(r.wr + (size_t)blockIdx.x * H);
        const uint64_t pol = l2_evict_last_policy();  // reused by every token
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = threadIdx.x + kRouteThreads * u;
            if (c < nch) wv[u] = ld_hint16(row + c, pol);
        }
    }
    if (kWhole && threadIdx.x < T * k) s_hmax[threadIdx.x] = 0u;
    if (threadIdx.x == 0) {
        ring_init(g, full, empty);
        if (kWhole) {
            mbar_init(&s_dbar, 1);
            mbar_fence_init();
        }
        // seq[b]: written by the CTA of the same index two launches back,
        // complete before this grid could start
        s_tag = ld_relaxed_gpu(r.hand.seq + blockIdx.x) + 1u;
    }
    __syncthreads();
    pdl_wait();  // the layer input comes from the previous kernel
    pdl_launch_dependents();
    const unsigned tag = s_tag;

    // ---- layer input -> routed vector (BF16, shared memory) ----
    if (rthread) {
        #pragma unroll 1
        for (int t = 0; t < T; ++t) {
            float s2 = 0.f, m = 0.f;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int c = threadIdx.x + kRouteThreads * u;
                if (c < nch) {
                    const uint4 v = reinterpret_cast<const uint4 *>(r.xr + (size_t)t * H)[c];
                    reinterpret_cast<uint4 *>(sx + (size_t)t * H)[c] = v;
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float a = bf16_to_f32(w4[q] & 0xFFFFu), b = bf16_to_f32(w4[q] >> 16);
                        s2 = fmaf(a, a, s2);
                        s2 = fmaf(b, b, s2);
                        m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
                    }
                }
            }
            s2 = warp_sum(s2);
            m = warp_max(m);
            if (lane == 0) {
                s_red[warp][t][0] = s2;
                s_red[warp][t][1] = m;
            }
        }
    }
    __syncthreads();
    // per token: 1 / RMS and the FP16 staging exponent of the routed vector;
    // max |BF16(x / rms)| = BF16(max|x| / rms) since rounding is monotone
    float inv[kDecodeMaxT];
#pragma unroll
    for (int tt = 0; tt < kDecodeMaxT; ++tt) {
        inv[tt] = 1.f;
        if (tt < T) {
            float a = 0.f, b = 0.f;
#pragma unroll
            for (int w = 0; w < kRouteWarps; ++w) {
                a += s_red[w][tt][0];
                b = fmaxf(b, s_red[w][tt][1]);
            }
            if (r.rmsnorm) {
                inv[tt] = 1.0f / sqrtf(a / (float)H + r.eps);
                b = round_bf16(b * inv[tt]);
            }
            if (threadIdx.x == 0) s_xexp[tt] = f16_stage_exponent(b);
        }
    }
    if (r.rmsnorm && rthread) {
        // weightless RMSNorm in place: xn = BF16(x / sqrt(mean(x^2) + eps)),
        // each thread on the pieces it loaded
        #pragma unroll 1
        for (int t = 0; t < T; ++t) {
            float iv = inv[0];
#pragma unroll
            for (int tt = 1; tt < kDecodeMaxT; ++tt)
                if (tt == t) iv = inv[tt];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int c = threadIdx.x + kRouteThreads * u;
                if (c < nch) {
                    uint4 *pv = reinterpret_cast<uint4 *>(sx + (size_t)t * H) + c;
                    const uint4 v = *pv;
                    uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        w4[q] = (uint32_t)f32_to_bf16(bf16_to_f32(w4[q] & 0xFFFFu) * iv) |
                                ((uint32_t)f32_to_bf16(bf16_to_f32(w4[q] >> 16) * iv) << 16);
                    const uint4 o = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    *pv = o;
                    if (blockIdx.x == 0 && r.x_norm)
                        reinterpret_cast<uint4 *>(r.x_norm + (size_t)t * H)[c] = o;
                }
            }
        }
    }
    __syncthreads();

    // ---- router: the logits of this CTA's experts, published as tagged words ----
    #pragma unroll 1
    for (int e = (int)blockIdx.x; e < E; e += G) {  // uniform over the CTA
        if (rthread) {
            if (e != (int)blockIdx.x) {
                const uint4 *row = reinterpret_cast<const uint4 *>(r.wr + (size_t)e * H);
                const uint64_t pol = l2_evict_last_policy();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = threadIdx.x + kRouteThreads * u;
                    wv[u] = c < nch ? ld_hint16(row + c, pol) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
            #pragma unroll 1
            for (int t = 0; t < T; ++t) {
                float acc = 0.f;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = threadIdx.x + kRouteThreads * u;
                    if (c < nch)
                        acc = dot8_bf16(reinterpret_cast<const uint4 *>(sx + (size_t)t * H)[c],
                                        wv[u], acc);
                }
                acc = warp_sum(acc);
                if (lane == 0) s_red[warp][t][0] = acc;
            }
        }
        __syncthreads();
        if (threadIdx.x < T) {
            const int t = threadIdx.x;
            float logit = 0.f;
#pragma unroll
            for (int w = 0; w < kRouteWarps; ++w) logit += s_red[w][t][0];
            if (r.bias) logit += r.bias[e];
            st_relaxed_gpu_v2(r.logit_ent + (size_t)t * E + e, tag, __float_as_uint(logit));
            if (r.logits_out) r.logits_out[(size_t)t * E + e] = logit;
        }
        __syncthreads();  // s_red is reused by the next expert
    }

    // down region (kWhole): staged h, expert outputs, the CTA's down rows
    const int I = p.I;
    const int R = dp.rows_per_cta;
    const int dr0 = (int)blockIdx.x * R, dr1 = min(dr0 + R, T * H);
    uint8_t *dreg = ring + dp.down_off;
    uint32_t *sh = reinterpret_cast<uint32_t *>(dreg);
    float *so = reinterpret_cast<float *>(dreg + (size_t)T * k * I * 2);
    uint8_t *rows_c = dreg + down_rows_offset(T, k, I, R);
    uint8_t *rows_s = rows_c + (size_t)k * R * ((size_t)I >> 1);
    const DownSrc src = {p.table, p.codes_base, p.scales_base, p.codes_stride, p.scales_stride};

    if (warp == kTmaConsumers) {
        // ---- producer warp: all logits, routing, the ring, and (with the
        // first copies in flight) the routing for the caller, the down rows
        // (kWhole) or the handoff to the down kernel ----
        if (!gather_logits(r.logit_ent, T * E, tag, s_logits) && lane == 0)
            atomicOr(p.status, kTimeoutStatus);
        __syncwarp();
        fused_topk(s_logits, T, E, k, s_ids, s_w);
        __syncwarp();
        ring_produce(p, g, ring, full, empty, s_ids, s_tab, lane, [&] {
            const int P = T * k;
            if (kWhole) {
                if (lane == 0)
                    issue_down_rows(src, E, H, I, k, s_ids, dr0, dr1, R, rows_c, rows_s, &s_dbar);
            } else {
                uint2 *ent = r.hand.ent + (size_t)blockIdx.x * kHandStride * 2;
                if (lane < P) {
                    st_relaxed_gpu_v2(ent + 2 * lane, tag, (unsigned)s_ids[lane]);
                    st_relaxed_gpu_v2(ent + 2 * lane + 1, tag, __float_as_uint(s_w[lane]));
                }
            }
            if (blockIdx.x == 0 && lane < P) {
                if (p.ids_out) p.ids_out[lane] = s_ids[lane];
                if (p.w_out) p.w_out[lane] = s_w[lane];
            }
            if (lane == 0) {
                st_relaxed_gpu(r.hand.seq + blockIdx.x, tag);
                // the down phase runs here: keep the handoff acknowledgement
                // in step for later two-launch calls on this workspace
                if (kWhole) st_relaxed_gpu(r.hand.ack + blockIdx.x, tag);
            }
        });
        if (!kWhole) return;
    } else {
        // ---- consumer warps: activations from the routed vector in shared memory ----
        ring_consume<KCH>(p, g, ring, full, empty, s_ids, warp, lane,
                          [&](int tok, uint32_t (&xw)[KCH][16]) -> float {
            const int c16 = s_xexp[tok];
            const float sf = pow2_neg(c16);
            const uint16_t *v = sx + (size_t)tok * H;
#pragma unroll
            for (int u = 0; u < KCH; ++u) {
                const int c = lane + 32 * u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 raw = c < C ? reinterpret_cast<const uint4 *>(v + (size_t)c * 32)[q]
                                            : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        xw[u][q * 4 + i] = f32x2_to_f16x2(bf16_to_f32(w4[i] & 0xFFFFu) * sf,
                                                          bf16_to_f32(w4[i] >> 16) * sf);
                }
            }
            return pow2(c16);
        }, [&](size_t idx, uint16_t v) {
            if (kWhole)
                st_relaxed_gpu_v2(dp.h_tag + idx, tag, v);
            else
                p.h[idx] = v;
        });
        if (!kWhole) return;
    }
    if constexpr (kWhole) {
        // ---- down phase: stage every h (tagged) -> the CTA's rows ----
        const int P = T * k;
        bool ok = stage_h_tagged(dp.h_tag, P, I, tag, sh, s_xs, s_hmax);
        if (!ok && threadIdx.x == 0) atomicOr(p.status, kTimeoutStatus);
        ok = __syncthreads_and(ok && mbar_wait(&s_dbar, 0u)) != 0;  // uniform over the CTA
        DownRows<TLD, KCHD, true> rows(H, I, k, E, R, dr0, dr1, src, s_ids, rows_c, rows_s);
        if (ok) rows.run(sh, s_xs, so, p.status);
        __syncthreads();
        if (ok) down_combine(dr0, dr1, H, k, R, so, s_w, dp.residual, dp.y, nullptr);
        // no row copy may outlive the CTA (complete unless its wait timed out)
        if (!ok && threadIdx.x == 0) mbar_wait(&s_dbar, 0u);
    }
}

// ------------------------------------------------------------------ host --

bool layer_gateup_plan(int T, int E, int H, int grid, size_t *smem, int *nslots,
                       unsigned *region_bytes) {
    if (T < 1 || T > kDecodeMaxT || E < 1 || E > kFusedMaxE) return false;
    if (grid < 1 || grid > kHandMaxCtas) return false;
    if (!gateup_tma_supported(H) || H > 2 * kRouteThreads * 8) return false;
    const size_t sx = (size_t)T * H * 2;
    const size_t slot = tma_slot_bytes(H);
    if (sx >= kFusedSmemBudget) return false;
    size_t n = (kFusedSmemBudget - sx) / slot;
    if (n > (size_t)kTmaMaxSlots) n = kTmaMaxSlots;
    if (n < 2) return false;
    const size_t region = (n * slot + 127) & ~(size_t)127;
    if (region + sx > kFusedSmemBudget) return false;
    *smem = region + sx;
    *nslots = (int)n;
    *region_bytes = (unsigned)region;
    return true;
}

bool layer_plan(int T, int E, int H, int I, int k, int grid, size_t *smem, int *nslots,
                unsigned *region_bytes, unsigned *down_off, int *rows_per_cta) {
    if (T < 1 || T > kDecodeMaxT || E < 1 || E > kFusedMaxE || k < 1 || k > kMaxTopK) return false;
    if (grid < 1 || grid > kHandMaxCtas) return false;
    if (!gateup_tma_supported(H) || H > 2048 || I % 512 != 0 || I > 4096) return false;
    if (kDownWarps < k) return false;
    const int R = (T * H + grid - 1) / grid;
    const size_t sx = (size_t)T * H * 2;
    const size_t down = down_rows_smem(T, k, I, R);
    const size_t slot = tma_slot_bytes(H);
    if (sx + down + 2 * slot > kFusedSmemBudget) return false;
    size_t n = (kFusedSmemBudget - sx - down - 128) / slot;
    if (n > (size_t)kTmaMaxSlots) n = kTmaMaxSlots;
    const size_t region = (n * slot + 127) & ~(size_t)127;
    const size_t doff = region + sx;  // 16-byte aligned: sx is a multiple of 1024
    if (doff + down > kFusedSmemBudget) return false;
    *smem = doff + down;
    *nslots = (int)n;
    *region_bytes = (unsigned)region;
    *down_off = (unsigned)doff;
    *rows_per_cta = R;
    return true;
}

namespace {

template <int KCH, int TLD, int KCHD>
cudaError_t launch_lk(const GateUpParams &p, const FusedRouteParams &r, const LayerDownParams &d,
                      int grid, size_t smem, cudaStream_t s, bool pdl) {
    // once per device (the attribute belongs to the current device's context)
    static PerDeviceOnce once;
    const cudaError_t smem_attr = per_device_once(once, [] {
        return cudaFuncSetAttribute(layer_kernel<KCH, TLD, KCHD>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kFusedSmemBudget);
    });
    if (smem_attr != cudaSuccess) return smem_attr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTmaThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    // One CTA per SM and grid = SM count: every CTA becomes resident as the
    // previous kernel's CTAs leave (nothing else runs on the stream), which the
    // logit polling and the done words rely on; the waits are bounded all the
    // same.  No cooperative attribute: it would hold every CTA back until the
    // whole GPU is free and lose the overlap with the previous kernel.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, layer_kernel<KCH, TLD, KCHD>, p, r, d);
}

template <int KCH>
cudaError_t launch_whole(const GateUpParams &p, const FusedRouteParams &r, const LayerDownParams &d,
                         int grid, size_t smem, cudaStream_t s, bool pdl) {
    int tl, kch;
    pick_team(p.I / 32, tl, kch);
    switch (tl * 10 + kch) {
    case 161: return launch_lk<KCH, 16, 1>(p, r, d, grid, smem, s, pdl);
    case 321: return launch_lk<KCH, 32, 1>(p, r, d, grid, smem, s, pdl);
    case 163: return launch_lk<KCH, 16, 3>(p, r, d, grid, smem, s, pdl);
    case 322: return launch_lk<KCH, 32, 2>(p, r, d, grid, smem, s, pdl);
    case 323: return launch_lk<KCH, 32, 3>(p, r, d, grid, smem, s, pdl);
    case 324: return launch_lk<KCH, 32, 4>(p, r, d, grid, smem, s, pdl);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_layer_gateup(const GateUpParams &p, const FusedRouteParams &r, int grid,
                                size_t smem, cudaStream_t s, bool pdl) {
    const LayerDownParams none = {};
    switch ((p.H / 32 + 31) / 32) {
    case 1: return launch_lk<1, 0, 0>(p, r, none, grid, smem, s, pdl);
    case 2: return launch_lk<2, 0, 0>(p, r, none, grid, smem, s, pdl);
    case 3: return launch_lk<3, 0, 0>(p, r, none, grid, smem, s, pdl);
    case 4: return launch_lk<4, 0, 0>(p, r, none, grid, smem, s, pdl);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_layer(const GateUpParams &p, const FusedRouteParams &r,
                         const LayerDownParams &d, int grid, size_t smem, cudaStream_t s,
                         bool pdl) {
    switch ((p.H / 32 + 31) / 32) {
    case 1: return launch_whole<1>(p, r, d, grid, smem, s, pdl);
    case 2: return launch_whole<2>(p, r, d, grid, smem, s, pdl);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
