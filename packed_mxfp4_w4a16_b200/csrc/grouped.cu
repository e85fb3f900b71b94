// grouped.cu — the (token, expert)-sorted grouped path of the packed-MXFP4
// W4A16 MoE expert FFN, for batches of tokens (prefill chunks, many decode
// streams).
//
// Sources: model card "LFM2.5-24B-A2B — Packed MXFP4 Inference", "Grouped
// top-4 expert execution" (grouped gate / up / down products, activation and
// multiplication, fused combine keeping sequential BF16 multiply/add
// rounding) and table "Model and quantization" (E2M1 + E8M0 per 32, BF16
// activations, FP32 accumulation); page "LFM2.5-8B-A1B — Core AI (.aimodel)",
// section "Provenance" (its batched SwitchGLU serves the 64-token prefill by
// sorting the (token, expert) pairs, so that each expert's tokens form one
// contiguous group before the quantized product).
//
// Launch sequence (one stream, programmatic serialization):
//   grouped_prep_kernel      CTA 0: stable counting sort of the T k (token,
//                            slot) pairs by expert -> perm, offs.  CTAs 1..T:
//                            FP16 staging of each token's activations.
//   grouped_mma_kernel<2>    per (expert, 16 gate/up rows): h = SwiGLU of the
//                            expert's tokens, on the tensor cores.
//   grouped_stage_h_kernel   per pair: FP16 staging of h.
//   grouped_mma_kernel<1>    per (expert, 16 down rows): o = BF16(W_down h).
//   grouped_combine_kernel   per token: sequential BF16 combine (+ residual).
// When the groups average at least kTcAutoGroup pairs (or on request) the
// two products and the h staging between them are replaced by the tcgen05
// kernels of grouped_tc.cu (BF16 tiles, TMEM accumulators).
//
// Tensor-core tile.  A CTA holds 16 packed rows of one expert matrix (codes
// and E8M0 scales; gate and up together) in shared memory and passes the
// expert's tokens through in chunks of 8 FP16-staged activation rows, all in
// row-padded layouts (conflict-free fragment loads).
// mma.m16n8k16 (FP16 x FP16 -> FP32) takes A = the E2M1 codes converted to
// FP16 in registers (exact) and B = the activations.  Within each 32-element
// group the K order is permuted identically for A and B so that each thread's
// A operand is one aligned 4-byte word of the row (8 codes) and its B operand
// one 16-byte piece of the activation row; the group's partial product (two
// MMAs, fresh accumulator) is then scaled by the group's E8M0 exponent in
// FP32 and added to the running FP32 sum, which is exactly per-group scaling.
// The K quarters (one per warp of a row tile) are added in a fixed order.
// The same tiles serve NVFP4 weights (page "primitive-ai/LFM2.5-24B-A2B-
// NVFP4A16": each 16-element block's partial product scaled by its E4M3
// scale) and sym8 weights (page "LFM2.5-8B-A1B — Core AI (.aimodel)",
// "Provenance": 8 int8 bytes per thread and row converted to FP16 exactly,
// the group's partial product scaled by its binary16 scale).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "gemv.cuh"

namespace moe {

namespace {

constexpr int kGpThreads = 256;   // prep / staging / combine CTAs
constexpr int kGpRows = 16;       // rows of one MMA row tile
constexpr int kGpMaxE = 1024;

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

__device__ __forceinline__ const uint8_t *mat_codes(const GroupedParams &p, int e, int m) {
    return p.codes_base ? p.codes_base + (size_t)(3 * e + m) * p.codes_stride : p.table[e].codes[m];
}
__device__ __forceinline__ const uint8_t *mat_scales(const GroupedParams &p, int e, int m) {
    return p.codes_base ? p.scales_base + (size_t)(3 * e + m) * p.scales_stride
                        : p.table[e].scales[m];
}

// FP16 staging of the BF16 vector v[0..n) (as the decode path stages it): the
// CTA's max |v| picks c, out = v 2^-c as f16x2 words; returns c.  All threads.
__device__ __forceinline__ int stage_vector_f16(const uint16_t *v, int n, uint32_t *out,
                                                float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int npc = n >> 3;  // 8-element pieces
    float m = 0.f;
    for (int c = threadIdx.x; c < npc; c += kGpThreads) {
        const uint4 x = reinterpret_cast<const uint4 *>(v)[c];
        const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            m = fmaxf(m, fmaxf(fabsf(bf16_to_f32(w4[q] & 0xFFFFu)), fabsf(bf16_to_f32(w4[q] >> 16))));
    }
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < kGpThreads / 32; ++i) amax = fmaxf(amax, red[i]);
    const int e = f16_stage_exponent(amax);
    const float sf = pow2_neg(e);
    for (int c = threadIdx.x; c < npc; c += kGpThreads) {
        const uint4 x = reinterpret_cast<const uint4 *>(v)[c];
        uint4 o;
        o.x = f32x2_to_f16x2(bf16_to_f32(x.x & 0xFFFFu) * sf, bf16_to_f32(x.x >> 16) * sf);
        o.y = f32x2_to_f16x2(bf16_to_f32(x.y & 0xFFFFu) * sf, bf16_to_f32(x.y >> 16) * sf);
        o.z = f32x2_to_f16x2(bf16_to_f32(x.z & 0xFFFFu) * sf, bf16_to_f32(x.z >> 16) * sf);
        o.w = f32x2_to_f16x2(bf16_to_f32(x.w & 0xFFFFu) * sf, bf16_to_f32(x.w >> 16) * sf);
        reinterpret_cast<uint4 *>(out)[c] = o;
    }
    return e;
}

}  // namespace

// ------------------------------------------------------------------ prep --
// CTA 0: stable counting sort of the pairs q = t k + j by expert (ties in pair
// order); invalid ids are left out of every segment and flag the status.
// CTAs 1..T: FP16 staging of token t = blockIdx.x - 1.
__global__ void __launch_bounds__(kGpThreads) grouped_prep_kernel(const GroupedParams p) {
    __shared__ int s_cnt[kGpMaxE];
    __shared__ float s_red[kGpThreads / 32];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (blockIdx.x > 0) {
        const int t = blockIdx.x - 1;
        const int c = stage_vector_f16(p.x + (size_t)t * p.H, p.H, p.x16 + (size_t)t * (p.H >> 1),
                                       s_red);
        if (threadIdx.x == 0) p.x_exp[t] = c;
        return;
    }
    const int E = p.E, P = p.T * p.k;
    for (int e = threadIdx.x; e < E; e += kGpThreads) s_cnt[e] = 0;
    __syncthreads();
    bool bad = false;
    for (int q = threadIdx.x; q < P; q += kGpThreads) {
        const int e = p.ids[q];
        if (e >= 0 && e < E)
            atomicAdd(&s_cnt[e], 1);
        else
            bad = true;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(p.status, kBadExpertId);
    if (warp == 0) {
        // exclusive scan: lane L sums a block of ceil(E/32) counts, the warp
        // scans the block sums, each lane then writes its block's starts
        const int per = (E + 31) / 32;
        const int b0 = min(E, lane * per), b1 = min(E, b0 + per);
        int sum = 0;
        for (int e = b0; e < b1; ++e) sum += s_cnt[e];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
        for (int e = b0; e < b1; ++e) {
            const int c = s_cnt[e];
            s_cnt[e] = run;  // becomes the next free slot of expert e
            p.offs[e] = run;
            run += c;
        }
        if (lane == 31) p.offs[E] = incl;
        __syncwarp();
        // placement in pair order, 32 pairs per round: the rank of a pair among
        // the round's pairs of the same expert comes from a match vote
        for (int base = 0; base < P; base += 32) {
            const int q = base + lane;
            const int e = q < P ? p.ids[q] : -1;
            const bool valid = e >= 0 && e < E;
            const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : E + lane);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            const int pos = valid ? s_cnt[e] + rank : 0;
            __syncwarp();
            if (valid && rank == 0) s_cnt[e] += __popc(peers);
            if (valid) p.perm[pos] = q;
            __syncwarp();
        }
    }
}

// -------------------------------------------------- tensor-core products --
// NMAT = 2: gate and up rows of expert blockIdx.y against the FP16-staged x
// of its tokens -> h (SwiGLU, BF16) of its pairs.  NMAT = 1: down rows
// against the staged h of its pairs -> o (BF16) of its pairs.
//
// One CTA per (RT row tiles of 16 rows, expert): the tiles' packed rows
// (codes and E8M0 scales of NMAT matrices) stay in shared memory while the
// expert's tokens pass through in chunks of 8 (the B tile).  Warp w works on
// row tile w / 4 and the (w % 4)-th quarter of the K groups; the quarters are
// added in a fixed order through shared memory and the quarter-0 warp of each
// tile writes its results.  Several CTAs per SM hide one another's copy and
// barrier latency.

constexpr int kRowTiles = 2;  // row tiles per CTA

template <int N>
__device__ __forceinline__ void cp_async_commit_wait() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group %0;" ::"n"(N) : "memory");
}

// NV: NVFP4 weights (two E4M3 scales per 32-element group, mma_group_nvfp4's
// K order; the expert's multiplier joins the power-of-two staging scale in the
// epilogue, an exact product).  S8: sym8 weights (one byte per weight, a
// binary16 scale per 32-element group, mma_group_s8).
template <int NMAT, int RT, bool NV, bool S8>
__global__ void __launch_bounds__(128 * RT) grouped_mma_kernel(const GroupedParams p) {
    constexpr int kWarps = 4 * RT;
    extern __shared__ __align__(16) uint8_t sm[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.y;
    pdl_wait();
    pdl_launch_dependents();
    const int seg0 = p.offs[e], n_e = p.offs[e + 1] - seg0;
    if (n_e <= 0) return;  // uniform: no token chose this expert

    const int K = NMAT == 2 ? p.H : p.I;  // reduction length
    const int M = NMAT == 2 ? p.I : p.H;  // rows of the matrix (a multiple of 16 RT)
    const int row0 = blockIdx.x * (kGpRows * RT);
    const int ng = K >> 5;                // 32-element groups
    // row bytes: codes (K/2 packed, K for sym8), scales (K/32 E8M0, K/16 for
    // E4M3 per 16 or binary16 per 32)
    const uint32_t rc = S8 ? (uint32_t)K : (uint32_t)K >> 1,
                   rs = (uint32_t)K >> (NV || S8 ? 4 : 5);
    const uint32_t rcp = rc + 16, rsp = rs + 16;  // padded row pitches (bank spread)
    const uint32_t bp = (uint32_t)K * 2 + 64;     // padded pitch of a staged B row
    constexpr int R = kGpRows * RT;               // rows held by the CTA
    uint8_t *s_codes = sm;                                      // [NMAT][R][rcp]
    uint8_t *s_scales = sm + NMAT * R * rcp;                    // [NMAT][R][rsp]
    float *s_red = reinterpret_cast<float *>(s_scales + NMAT * R * rsp);
    // s_red: [RT][3 quarters][32 lanes][NMAT * 4] partial sums
    uint8_t *s_b = reinterpret_cast<uint8_t *>(s_red + RT * 3 * 32 * NMAT * 4);  // [8][bp]

    // ---- the CTA's rows of each matrix into shared memory ----
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
        const int mat = NMAT == 2 ? m : 2;
        const uint8_t *gc = mat_codes(p, e, mat) + (size_t)row0 * rc;
        const uint8_t *gs = mat_scales(p, e, mat) + (size_t)row0 * rs;
        const int c16 = (int)(rc >> 4), c4 = (int)(rs >> 2);
        for (int r = warp; r < R; r += kWarps) {
            uint8_t *dc = s_codes + (m * R + r) * rcp;
            uint8_t *ds = s_scales + (m * R + r) * rsp;
            for (int c = lane; c < c16; c += 32) cp_async16(dc + c * 16, gc + r * rc + c * 16);
            for (int c = lane; c < c4; c += 32) cp_async4(ds + c * 4, gs + r * rs + c * 4);
        }
    }
    // B: the staged FP16 vectors of up to 8 tokens (x of the pair's token for
    // gate / up, h of the pair for down); the columns of absent tokens hold
    // whatever the buffer held and only feed results that are not written
    const int cb16 = K >> 3;
    auto stage_b = [&](int tc) {
        for (int tk = warp; tk < 8; tk += kWarps) {
            const int idx = tc + tk;
            if (idx >= n_e) break;
            const int pr = p.perm[seg0 + idx];
            const uint8_t *src = reinterpret_cast<const uint8_t *>(
                NMAT == 2 ? p.x16 + (size_t)(pr / p.k) * (K >> 1) : p.h16 + (size_t)pr * (K >> 1));
            uint8_t *dst = s_b + tk * bp;
            for (int c = lane; c < cb16; c += 32) cp_async16(dst + c * 16, src + c * 16);
        }
    };
    stage_b(0);
    cp_async_commit_wait<0>();
    __syncthreads();

    const int g = lane >> 2, q = lane & 3;
    const int rt = warp >> 2, kq = warp & 3;  // row tile, K quarter
    const int gq = (ng + 3) >> 2;
    const int gb = min(ng, kq * gq), ge = min(ng, gb + gq);
    // this thread's A words (rows g / g + 8 of its tile) and scales
    const uint8_t *a_lo = s_codes + (rt * kGpRows + g) * rcp + (NV ? 2 * q : S8 ? 8 * q : 4 * q);
    const uint8_t *s_lo = s_scales + (rt * kGpRows + g) * rsp;
    const uint32_t a_hi = 8 * rcp, sc_hi = 8 * rsp;
    const uint32_t a_m = R * rcp, sc_m = R * rsp;
    // column g = token tc + g of the group
    const uint8_t *bcol = s_b + g * bp + (NV ? 8 * q : 16 * q);

    #pragma unroll 1
    for (int tc = 0; tc < n_e; tc += 8) {
        if (tc > 0) {
            stage_b(tc);
            cp_async_commit_wait<0>();
            __syncthreads();
        }
        float acc[NMAT][4];
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;

        #pragma unroll 4
        for (int G = gb; G < ge; ++G) {
            if (NV) {
                // block 0 elements 4q..4q+3, then block 1's
                const uint2 b0 = *reinterpret_cast<const uint2 *>(bcol + G * 64);
                const uint2 b1 = *reinterpret_cast<const uint2 *>(bcol + G * 64 + 32);
                const uint4 b = make_uint4(b0.x, b0.y, b1.x, b1.y);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint8_t *cb = a_lo + m * a_m + G * 16;
                    const uint16_t *sb = reinterpret_cast<const uint16_t *>(s_lo + m * sc_m + 2 * G);
                    const uint32_t wl = *reinterpret_cast<const uint16_t *>(cb) |
                                        ((uint32_t)*reinterpret_cast<const uint16_t *>(cb + 8) << 16);
                    const uint32_t wh = *reinterpret_cast<const uint16_t *>(cb + a_hi) |
                                        ((uint32_t)*reinterpret_cast<const uint16_t *>(cb + a_hi + 8) << 16);
                    mma_group_nvfp4(acc[m], wl, wh, sb[0],
                                    *reinterpret_cast<const uint16_t *>(
                                        reinterpret_cast<const uint8_t *>(sb) + sc_hi),
                                    b);
                }
            } else if (S8) {
                const uint4 b = *reinterpret_cast<const uint4 *>(bcol + G * 64);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint8_t *cb = a_lo + m * a_m + G * 32;
                    const uint8_t *sb = s_lo + m * sc_m + 2 * G;
                    mma_group_s8(acc[m], *reinterpret_cast<const uint2 *>(cb),
                                 *reinterpret_cast<const uint2 *>(cb + a_hi),
                                 *reinterpret_cast<const uint16_t *>(sb),
                                 *reinterpret_cast<const uint16_t *>(sb + sc_hi), b);
                }
            } else {
                const uint4 b = *reinterpret_cast<const uint4 *>(bcol + G * 64);
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const uint8_t *cb = a_lo + m * a_m + G * 16;
                    const uint8_t *sb = s_lo + m * sc_m + G;
                    mma_group_e2m1(acc[m], *reinterpret_cast<const uint32_t *>(cb),
                                   *reinterpret_cast<const uint32_t *>(cb + a_hi), sb[0], sb[sc_hi], b);
                }
            }
        }
        // ---- the 4 K quarters of each row tile, added in order 0, 1, 2, 3 ----
        float *red = s_red + rt * (3 * 32 * NMAT * 4);
        if (kq > 0) {
            float *dst = red + ((kq - 1) * 32 + lane) * (NMAT * 4);
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[m * 4 + i] = acc[m][i];
        }
        __syncthreads();
        if (kq == 0) {
#pragma unroll
            for (int qq = 1; qq < 4; ++qq) {
                const float *src = red + ((qq - 1) * 32 + lane) * (NMAT * 4);
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[m][i] += src[m * 4 + i];
            }
            // ---- epilogue: rows g / g + 8 of the tile, columns (tokens) 2q, 2q + 1 ----
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int idx = tc + 2 * q + cc;
                if (idx >= n_e) continue;
                const int pr = p.perm[seg0 + idx];
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int r = row0 + rt * kGpRows + g + 8 * hr;
                    if (NMAT == 2) {
                        const float xs = NV ? pow2(p.x_exp[pr / p.k]) * __ldg(p.gscale + 2 * e)
                                            : pow2(p.x_exp[pr / p.k]);
                        const float gv = round_bf16(acc[0][hr * 2 + cc] * xs);
                        const float uv = round_bf16(acc[NMAT - 1][hr * 2 + cc] * xs);
                        const float sl = round_bf16(gv / (1.0f + expf(-gv)));
                        p.h[(size_t)pr * M + r] = f32_to_bf16(sl * uv);
                    } else {
                        const float hs = NV ? pow2(p.h_exp[pr]) * __ldg(p.gscale + 2 * e + 1)
                                            : pow2(p.h_exp[pr]);
                        p.o[(size_t)pr * M + r] = f32_to_bf16(acc[0][hr * 2 + cc] * hs);
                    }
                }
            }
        }
        if (tc + 8 < n_e) __syncthreads();  // s_red and s_b are reused by the next chunk
    }
}

// ------------------------------------------------------------- stage h --
__global__ void __launch_bounds__(kGpThreads) grouped_stage_h_kernel(const GroupedParams p) {
    __shared__ float s_red[kGpThreads / 32];
    pdl_wait();
    pdl_launch_dependents();
    const int pr = blockIdx.x;
    const int e = p.ids[pr];
    if (e < 0 || e >= p.E) return;  // uniform: the pair has no h
    const int c = stage_vector_f16(p.h + (size_t)pr * p.I, p.I, p.h16 + (size_t)pr * (p.I >> 1),
                                   s_red);
    if (threadIdx.x == 0) p.h_exp[pr] = c;
}

// ------------------------------------------------------------- combine --
// y[t] = sequential BF16 combine of the k expert outputs in slot order (a pair
// with an invalid id contributes 0), then the optional residual add.
__global__ void __launch_bounds__(kGpThreads) grouped_combine_kernel(const GroupedParams p) {
    pdl_wait();
    pdl_launch_dependents();
    const int t = blockIdx.x, k = p.k, H = p.H;
    // the token's slots: expert ids (validity) and BF16-rounded weights, read
    // once, before the expert output rows (k <= kMaxTopK)
    bool ok[kMaxTopK];
    float wb[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        const int e = j < k ? p.ids[t * k + j] : -1;
        ok[j] = e >= 0 && e < p.E;
        wb[j] = j < k ? round_bf16(p.w[t * k + j]) : 0.f;
    }
    // 8 consecutive elements per thread (H is a multiple of 128)
    for (int c = threadIdx.x; c < (H >> 3); c += kGpThreads) {
        uint4 ov[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
            ov[j] = (j < k && ok[j])
                        ? reinterpret_cast<const uint4 *>(p.o + (size_t)(t * k + j) * H)[c]
                        : make_uint4(0u, 0u, 0u, 0u);
        uint4 rv = make_uint4(0u, 0u, 0u, 0u);
        if (p.residual) rv = reinterpret_cast<const uint4 *>(p.residual + (size_t)t * H)[c];
        const uint32_t *rw = &rv.x;
        uint32_t out[4];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float y = 0.f;
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j >= k) break;
                const uint32_t word = (&ov[j].x)[i >> 1];
                const float o = bf16_to_f32((i & 1) ? word >> 16 : word & 0xFFFFu);
                y = round_bf16(y + round_bf16(o * wb[j]));
            }
            if (p.residual) {
                const uint32_t word = rw[i >> 1];
                y = round_bf16(bf16_to_f32((i & 1) ? word >> 16 : word & 0xFFFFu) + y);
            }
            const uint32_t b = f32_to_bf16(y);
            out[i >> 1] = (i & 1) ? (out[i >> 1] | (b << 16)) : b;
        }
        reinterpret_cast<uint4 *>(p.y + (size_t)t * H)[c] = make_uint4(out[0], out[1], out[2], out[3]);
        if (p.o_keep) {
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j)
                if (j < k) reinterpret_cast<uint4 *>(p.o_keep + (size_t)(t * k + j) * H)[c] = ov[j];
        }
    }
}

// ------------------------------------------------------------------ host --

namespace {

constexpr size_t kMmaSmemBudget = 220 * 1024;

// row tiles per CTA of the sym8 products (their rows take twice the bytes)
#ifndef MOE_S8_GROUPED_RT
#define MOE_S8_GROUPED_RT 1
#endif
constexpr int kS8RowTiles = MOE_S8_GROUPED_RT;

size_t mma_smem(int nmat, int K, int nv, int s8) {
    const int rt = s8 ? kS8RowTiles : kRowTiles;
    const size_t R = (size_t)kGpRows * rt;
    const size_t rcp = (size_t)K / (s8 ? 1 : 2) + 16,
                 rsp = (size_t)K / (nv || s8 ? 16 : 32) + 16;
    return (size_t)nmat * R * (rcp + rsp) + (size_t)rt * 3 * 32 * nmat * 4 * sizeof(float) +
           (size_t)8 * ((size_t)K * 2 + 64);
}

template <int NMAT, bool NV, bool S8>
cudaError_t launch_mma(const GroupedParams &p, cudaStream_t s, bool pdl) {
    constexpr int RT = S8 ? kS8RowTiles : kRowTiles;
    const int K = NMAT == 2 ? p.H : p.I, M = NMAT == 2 ? p.I : p.H;
    const size_t smem = mma_smem(NMAT, K, NV ? 1 : 0, S8 ? 1 : 0);
    if (smem > kMmaSmemBudget) return cudaErrorInvalidValue;
    // the budget, once per device (the attribute belongs to the current
    // device's context)
    static PerDeviceOnce once;
    const cudaError_t attr = per_device_once(once, [] {
        return cudaFuncSetAttribute(grouped_mma_kernel<NMAT, RT, NV, S8>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kMmaSmemBudget);
    });
    if (attr != cudaSuccess) return attr;
    return launch_ex(grouped_mma_kernel<NMAT, RT, NV, S8>, dim3(M / (kGpRows * RT), p.E),
                     dim3(128 * RT), smem, s, pdl, p);
}

}  // namespace

bool grouped_supported(int E, int H, int I, int nv, int s8) {
    // the pipeline stages of both products must fit the shared memory budget
    return E <= kGpMaxE && H % 128 == 0 && I % 128 == 0 && H <= 4096 && I <= 4096 &&
           !(nv && s8) && mma_smem(2, H, nv, s8) <= kMmaSmemBudget &&
           mma_smem(1, I, nv, s8) <= kMmaSmemBudget;
}

cudaError_t launch_grouped(const GroupedParams &p, cudaStream_t s, bool pdl) {
    if (p.T < 1 || p.T > kGroupedMaxT || !grouped_supported(p.E, p.H, p.I, p.nv, p.s8))
        return cudaErrorInvalidValue;
    if (p.tcgen05 &&
        (p.s8 || !p.codes_base || !grouped_tc_supported(p.H, p.I, p.nv)))
        return cudaErrorInvalidValue;
    if (p.nv && !p.gscale) return cudaErrorInvalidValue;
    cudaError_t e;
    if ((e = launch_ex(grouped_prep_kernel, dim3(p.T + 1), dim3(kGpThreads), 0, s, pdl, p)) !=
        cudaSuccess)
        return e;
    if (p.tcgen05) {
        // the products on tcgen05 (BF16 tiles, TMEM accumulators; they read
        // x and h in BF16, so h needs no FP16 staging)
        if ((e = launch_grouped_tc_gateup(p, s, pdl)) != cudaSuccess) return e;
        if ((e = launch_grouped_tc_down(p, s, pdl)) != cudaSuccess) return e;
    } else {
        if ((e = p.s8   ? launch_mma<2, false, true>(p, s, pdl)
                 : p.nv ? launch_mma<2, true, false>(p, s, pdl)
                        : launch_mma<2, false, false>(p, s, pdl)) != cudaSuccess)
            return e;
        if ((e = launch_ex(grouped_stage_h_kernel, dim3(p.T * p.k), dim3(kGpThreads), 0, s, pdl,
                           p)) != cudaSuccess)
            return e;
        if ((e = p.s8   ? launch_mma<1, false, true>(p, s, pdl)
                 : p.nv ? launch_mma<1, true, false>(p, s, pdl)
                        : launch_mma<1, false, false>(p, s, pdl)) != cudaSuccess)
            return e;
    }
    return launch_ex(grouped_combine_kernel, dim3(p.T), dim3(kGpThreads), 0, s, pdl, p);
}


}  // namespace moe
