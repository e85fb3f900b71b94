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

// ------------------------------------------------------------------ route --

__global__ void __launch_bounds__(kRouteThreads)
route_kernel(const RouteParams p) {
    extern __shared__ float xs[];  // [H] the routed vector in FP32
    __shared__ float s_red[kRouteThreads / 32];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.y, H = p.H, E = p.E, k = p.k;
    const uint16_t *xt = p.x + (size_t)t * H;

    pdl_wait();
    pdl_launch_dependents();

    if (p.rmsnorm) {
        // weightless RMSNorm: xn = BF16(r / sqrt(mean(r^2) + eps))
        float ss = 0.f;
        for (int i = tid; i < H; i += kRouteThreads) {
            float v = bf16_to_f32(xt[i]);
            ss = fmaf(v, v, ss);
        }
        ss = warp_sum(ss);
        if (lane == 0) s_red[warp] = ss;
        __syncthreads();
        if (warp == 0) {
            float v = lane < kRouteThreads / 32 ? s_red[lane] : 0.f;
            v = warp_sum(v);
            if (lane == 0) s_red[0] = 1.0f / sqrtf(v / (float)H + p.eps);
        }
        __syncthreads();
        const float inv = s_red[0];
        for (int i = tid; i < H; i += kRouteThreads) {
            uint16_t b = f32_to_bf16(bf16_to_f32(xt[i]) * inv);
            xs[i] = bf16_to_f32(b);
            if (blockIdx.x == 0) p.x_norm[(size_t)t * H + i] = b;
        }
    } else {
        for (int i = tid; i < H; i += kRouteThreads) xs[i] = bf16_to_f32(xt[i]);
    }
    __syncthreads();

    // one expert row per warp: logits = x . Wr[e] in FP32 (+ bias)
    const int nchunk = H >> 3;  // 8 BF16 per 16-byte chunk
    for (int e = blockIdx.x * (kRouteThreads / 32) + warp; e < E;
         e += gridDim.x * (kRouteThreads / 32)) {
        const uint16_t *row = p.wr + (size_t)e * H;
        float acc = 0.f;
        for (int c = lane; c < nchunk; c += 32) {
            uint4 v = *reinterpret_cast<const uint4 *>(row + (size_t)c * 8);
            const float *xv = xs + c * 8;
            acc = fmaf(bf16_to_f32(v.x & 0xFFFFu), xv[0], acc);
            acc = fmaf(bf16_to_f32(v.x >> 16), xv[1], acc);
            acc = fmaf(bf16_to_f32(v.y & 0xFFFFu), xv[2], acc);
            acc = fmaf(bf16_to_f32(v.y >> 16), xv[3], acc);
            acc = fmaf(bf16_to_f32(v.z & 0xFFFFu), xv[4], acc);
            acc = fmaf(bf16_to_f32(v.z >> 16), xv[5], acc);
            acc = fmaf(bf16_to_f32(v.w & 0xFFFFu), xv[6], acc);
            acc = fmaf(bf16_to_f32(v.w >> 16), xv[7], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) {
            if (p.bias) acc += p.bias[e];
            p.logits_ws[(size_t)t * E + e] = acc;
        }
    }

    // the last CTA of this token selects (no waiting: an arrival counter)
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        unsigned prev = atomicAdd(p.counters + t, 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last || warp != 0) return;
    __threadfence();

    const float *lg = p.logits_ws + (size_t)t * E;
    int chosen[kMaxTopK];
    float chosen_v[kMaxTopK];
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7FFFFFFF;
        for (int e = lane; e < E; e += 32) {
            bool taken = false;
            for (int q = 0; q < j; ++q) taken |= (chosen[q] == e);
            float v = __ldcg(lg + e);
            if (!taken && (v > bv || (v == bv && e < bi))) {
                bv = v;
                bi = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        chosen[j] = bi;
        chosen_v[j] = bv;
    }
    if (lane == 0) {
        // coefficients: softmax over the k selected logits (slot 0 is the max)
        float z = 0.f, ex[kMaxTopK];
        for (int j = 0; j < k; ++j) {
            ex[j] = expf(chosen_v[j] - chosen_v[0]);
            z += ex[j];
        }
        for (int j = 0; j < k; ++j) {
            p.ids[(size_t)t * k + j] = chosen[j];
            p.w[(size_t)t * k + j] = ex[j] / z;
        }
        p.counters[t] = 0u;
    }
    if (p.logits_out)
        for (int e = lane; e < E; e += 32) p.logits_out[(size_t)t * E + e] = __ldcg(lg + e);
}

// --------------------------------------------------------------- staging --

// Stage BF16 vector v[0..n) as FP16 words in shared memory (scaled by 2^-c,
// c from the vector's max |v|); returns c.  Called by one warp.
__device__ __forceinline__ int stage_f16_warp(const uint16_t *v, int n, uint32_t *dst,
                                              int lane) {
    float m = 0.f;
    const uint32_t *v2 = reinterpret_cast<const uint32_t *>(v);
    for (int i = lane; i < (n >> 1); i += 32) {
        uint32_t pr = v2[i];
        m = fmaxf(m, fmaxf(fabsf(bf16_to_f32(pr & 0xFFFFu)), fabsf(bf16_to_f32(pr >> 16))));
    }
    m = warp_max(m);
    const int c = f16_stage_exponent(m);
    for (int i = lane; i < (n >> 1); i += 32) {
        uint32_t pr = v2[i];
        float a = scalbnf(bf16_to_f32(pr & 0xFFFFu), -c);
        float b = scalbnf(bf16_to_f32(pr >> 16), -c);
        dst[i] = (uint32_t)f32_to_f16_bits(a) | ((uint32_t)f32_to_f16_bits(b) << 16);
    }
    return c;
}

// Sum over the KCH chunks of one lane of a packed row against staged FP16
// activations (xw = the row's activation words).  Each chunk is one E8M0 group.
template <int TL, int KCH>
__device__ __forceinline__ float row_partial(const uint4 (&cw)[KCH], const uint32_t (&sc)[KCH],
                                             const uint32_t *xw, int lt, int C) {
    float acc = 0.f;
#pragma unroll
    for (int m = 0; m < KCH; ++m) {
        const int c = lt + m * TL;
        if (c < C) {
            const uint4 *xv = reinterpret_cast<const uint4 *>(xw + c * 16);
            uint32_t x[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 v = xv[q];
                x[4 * q + 0] = v.x;
                x[4 * q + 1] = v.y;
                x[4 * q + 2] = v.z;
                x[4 * q + 3] = v.w;
            }
            acc = fmaf(dot32_e2m1_f16(cw[m], x), e8m0_to_f32(sc[m]), acc);
        }
    }
    return acc;
}

template <int TL, int KCH>
__device__ __forceinline__ void load_row(const uint8_t *codes, const uint8_t *scales, bool ok,
                                         int lt, int C, uint4 (&cw)[KCH], uint32_t (&sc)[KCH]) {
#pragma unroll
    for (int m = 0; m < KCH; ++m) {
        const int c = lt + m * TL;
        if (ok && c < C) {
            cw[m] = ld_stream16(codes + (size_t)c * 16);
            sc[m] = ld_stream_u8(scales + c);
        } else {
            cw[m] = make_uint4(0u, 0u, 0u, 0u);
            sc[m] = 127u;
        }
    }
}

// ----------------------------------------------------------- gate / up ----

// L2 prefetch of this CTA's share of the selected experts' down matrices, so
// that the down GEMV that follows reads them from L2 while the DRAM keeps
// streaming.  Experts repeated across (token, slot) pairs are fetched once.
__device__ void prefetch_down_share(const GateUpParams &p) {
    const int P = p.T * p.k;
    const size_t mc = (size_t)p.H * p.I / 2, ms = (size_t)p.H * p.I / 32;
    for (int which = 0; which < 2; ++which) {
        const size_t per = which ? ms : mc;
        const size_t total = per * (size_t)P;
        const size_t b0 = (total * blockIdx.x / gridDim.x) & ~(size_t)15;
        const size_t b1 = (blockIdx.x + 1 == gridDim.x) ? total
                                                         : ((total * (blockIdx.x + 1) / gridDim.x) & ~(size_t)15);
        for (size_t b = b0; b < b1;) {
            const int q = (int)(b / per);
            const size_t off = b - (size_t)q * per;
            const size_t len = min(b1 - b, per - off);
            const int e = p.ids[q];
            bool dup = false;
            for (int q2 = 0; q2 < q; ++q2) dup |= (p.ids[q2] == e);
            if (!dup && e >= 0 && e < p.E) {
                const uint8_t *base = (which ? p.table[e].scales[2] : p.table[e].codes[2]) + off;
                for (size_t o = 0; o < len; o += 32768) {
                    const uint32_t n = (uint32_t)min((size_t)32768, len - o);
                    if (n >= 16) prefetch_l2_bulk(base + o, n & ~15u);
                }
            }
            b += len;
        }
    }
}

template <int TL, int KCH>
__global__ void __launch_bounds__(kGemvThreads, 1)
gateup_decode_kernel(const GateUpParams p) {
    extern __shared__ __align__(16) uint32_t sx[];  // [T][H/2] FP16 words
    __shared__ int s_c[kDecodeMaxT];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, I = p.I, k = p.k, T = p.T;
    const int C = H >> 5, hw = H >> 1;

    pdl_wait();  // x and ids come from earlier kernels
    pdl_launch_dependents();

    if (p.prefetch_down && tid == 0) prefetch_down_share(p);

    for (int t = warp; t < T; t += kGemvWarps) {
        int c = stage_f16_warp(p.x + (size_t)t * H, H, sx + (size_t)t * hw, lane);
        if (lane == 0) s_c[t] = c;
    }
    __syncthreads();

    // items (pair q = t*k + j, row i), q-major; each warp owns a contiguous
    // range, its 32/TL teams take items round-robin, two at a time.
    constexpr int TPW = 32 / TL;
    const int lt = lane % TL, tw = lane / TL;
    const long long N = (long long)T * k * I;
    const long long gw = (long long)blockIdx.x * kGemvWarps + warp;
    const long long GW = (long long)gridDim.x * kGemvWarps;
    const long long wb = N * gw / GW, we = N * (gw + 1) / GW;

    for (long long base = wb; base < we; base += 2 * TPW) {
        long long item[2] = {base + tw, base + TPW + tw};
        uint4 cg[2][KCH], cu[2][KCH];
        uint32_t sg[2][KCH], su[2][KCH];
        int q[2], row[2], tok[2];
        bool valid[2], bad[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            valid[u] = item[u] < we;
            q[u] = valid[u] ? (int)(item[u] / I) : 0;
            row[u] = valid[u] ? (int)(item[u] - (long long)q[u] * I) : 0;
            tok[u] = q[u] / k;
            int e = valid[u] ? p.ids[q[u]] : 0;
            bad[u] = valid[u] && (e < 0 || e >= p.E);
            const bool ok = valid[u] && !bad[u];
            const uint8_t *gc = nullptr, *gs = nullptr, *uc = nullptr, *us = nullptr;
            if (ok) {
                const ExpertPtrs *ep = p.table + e;
                gc = ep->codes[0] + (size_t)row[u] * (H >> 1);
                gs = ep->scales[0] + (size_t)row[u] * (H >> 5);
                uc = ep->codes[1] + (size_t)row[u] * (H >> 1);
                us = ep->scales[1] + (size_t)row[u] * (H >> 5);
            }
            load_row<TL, KCH>(gc, gs, ok, lt, C, cg[u], sg[u]);
            load_row<TL, KCH>(uc, us, ok, lt, C, cu[u], su[u]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t *xw = sx + (size_t)tok[u] * hw;
            float ag = row_partial<TL, KCH>(cg[u], sg[u], xw, lt, C);
            float au = row_partial<TL, KCH>(cu[u], su[u], xw, lt, C);
            ag = team_sum<TL>(ag);
            au = team_sum<TL>(au);
            if (lt == 0 && valid[u]) {
                uint16_t out = 0;
                if (!bad[u]) {
                    const int c = s_c[tok[u]];
                    const float g = round_bf16(scalbnf(ag, c));
                    const float uu = round_bf16(scalbnf(au, c));
                    const float s = round_bf16(g / (1.0f + expf(-g)));
                    out = f32_to_bf16(s * uu);
                } else {
                    atomicOr(p.status, kBadExpertId);
                }
                p.h[(size_t)q[u] * I + row[u]] = out;
            }
        }
    }
}

// ---------------------------------------------------------------- down -----

template <int TL, int KCH>
__global__ void __launch_bounds__(kGemvThreads, 1)
down_decode_kernel(const DownParams p) {
    extern __shared__ __align__(16) uint32_t sd[];
    __shared__ int s_c[kDecodeMaxT * kMaxTopK];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H, I = p.I, k = p.k, T = p.T;
    const int P = T * k, C = I >> 5, iw = I >> 1;
    const int R = p.rows_per_cta;
    uint32_t *sh = sd;                                    // [P][I/2] FP16 words
    float *so = reinterpret_cast<float *>(sd + (size_t)P * iw);  // [k][R]

    pdl_wait();  // h comes from the gate/up kernel
    pdl_launch_dependents();

    for (int q = warp; q < P; q += kGemvWarps) {
        int c = stage_f16_warp(p.h + (size_t)q * I, I, sh + (size_t)q * iw, lane);
        if (lane == 0) s_c[q] = c;
    }
    __syncthreads();

    const int r0 = blockIdx.x * R;
    const int r1 = min(r0 + R, T * H);
    constexpr int TPW = 32 / TL;
    const int groups = kGemvWarps / k;  // warps per slot
    const int j = warp % k, gi = warp / k;
    const int lt = lane % TL, tw = lane / TL;
    const int tps = groups * TPW;       // teams per slot
    const int ti = gi * TPW + tw;

    if (gi < groups && r0 < r1) {
        for (int base = r0; base < r1; base += 2 * tps) {
            int rr[2] = {base + ti, base + tps + ti};
            uint4 cw[2][KCH];
            uint32_t sc[2][KCH];
            int qq[2];
            bool valid[2], bad[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                valid[u] = rr[u] < r1;
                const int t = valid[u] ? rr[u] / H : 0;
                const int n = rr[u] - t * H;
                qq[u] = t * k + j;
                const int e = valid[u] ? p.ids[qq[u]] : 0;
                bad[u] = valid[u] && (e < 0 || e >= p.E);
                const bool ok = valid[u] && !bad[u];
                const uint8_t *dc = nullptr, *ds = nullptr;
                if (ok) {
                    const ExpertPtrs *ep = p.table + e;
                    dc = ep->codes[2] + (size_t)n * (I >> 1);
                    ds = ep->scales[2] + (size_t)n * (I >> 5);
                }
                load_row<TL, KCH>(dc, ds, ok, lt, C, cw[u], sc[u]);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float a = row_partial<TL, KCH>(cw[u], sc[u], sh + (size_t)qq[u] * iw, lt, C);
                a = team_sum<TL>(a);
                if (lt == 0 && valid[u]) {
                    float o = 0.f;
                    if (!bad[u])
                        o = round_bf16(scalbnf(a, s_c[qq[u]]));
                    else
                        atomicOr(p.status, kBadExpertId);
                    so[j * R + (rr[u] - r0)] = o;
                }
            }
        }
    }
    __syncthreads();

    // sequential BF16 combine in slot order, optional residual add
    for (int r = r0 + tid; r < r1; r += kGemvThreads) {
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

constexpr size_t kMaxSmem = kMaxDecodeSmem;

template <int TL, int KCH>
cudaError_t launch_gu(const GateUpParams &p, int grid, cudaStream_t s, bool pdl) {
    auto kern = gateup_decode_kernel<TL, KCH>;
    size_t smem = gateup_decode_smem(p.T, p.H);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(grid), dim3(kGemvThreads), smem, s, pdl, p);
}

template <int TL, int KCH>
cudaError_t launch_dn(const DownParams &p, int grid, cudaStream_t s, bool pdl) {
    auto kern = down_decode_kernel<TL, KCH>;
    size_t smem = down_decode_smem(p.T, p.k, p.I, p.rows_per_cta);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3(grid), dim3(kGemvThreads), smem, s, pdl, p);
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

size_t gateup_decode_smem(int T, int H) { return (size_t)T * H * 2; }

size_t down_decode_smem(int T, int k, int I, int rows_per_cta) {
    return (size_t)T * k * I * 2 + (size_t)k * rows_per_cta * 4;
}

cudaError_t launch_route(const RouteParams &p, cudaStream_t s, bool pdl) {
    const int wpb = kRouteThreads / 32;
    const int nblk = (p.E + wpb - 1) / wpb;
    size_t smem = (size_t)p.H * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kMaxSmem);
    if (e != cudaSuccess) return e;
    return launch_ex(route_kernel, dim3(nblk, p.T), dim3(kRouteThreads), smem, s, pdl, p);
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
