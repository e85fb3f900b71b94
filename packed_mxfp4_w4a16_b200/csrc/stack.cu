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
// reader that sees this step's tag also sees the value written with it.  The
// words sit one 4-word piece (or one router logit) per 128-byte line, so the
// polls of ~150 CTAs spread over as many L2 lines as there are pieces.  Every
// wait is bounded.
//
// Weight formats: MXFP4 (E8M0 scale per 32) or, with NV, NVFP4 (two E4M3
// scales per 32-element chunk, each 16-element half sum scaled in FP32; the
// expert's FP32 gate/up and down multipliers folded into the power-of-two
// staging scales), one format per stack.
//
// One layer, CTA b of G:
//   A  the layer input r (the previous layer's tagged outputs, or the input
//      buffer for layer 0) into shared memory; weightless RMSNorm
//      xn = BF16(r / sqrt(mean(r^2) + 1e-6)); FP16 staging of xn for the GEMVs;
//      CTA b < E also computes router logit b (its router row was copied into
//      shared memory one layer ahead) and publishes it.
//   C  (producer warp) gathers all E logits, top-k + softmax; then ONE lane
//      requests with bulk copies all of the CTA's weight bytes of the layer,
//      in the order they are needed: the gate/up scales, the gate/up code
//      rows in a few pieces (one mbarrier each, so the GEMVs start when the
//      first piece lands), the CTA's output rows of the down matrices (one
//      mbarrier); another lane requests the next layer's router row.  The
//      whole layer's ~20 MB is in flight from here on.
//   D  (all warps) pairs of gate/up rows per warp from shared memory: E2M1
//      codes decoded in registers against the FP16 activations, FP32 sums,
//      SwiGLU, the two h values published as one tagged word.
//   E  kHThreads threads gather all of h (tagged) and stage it in shared
//      memory as FP16 (per-vector power of two).
//   F  the down GEMV of the CTA's output rows for every slot (rows already in
//      shared memory), by lane teams two rows at a time, each chunk of h
//      loaded once for both rows.
//   G  sequential BF16 combine in slot order and the residual add; the layer
//      output rows are published as tagged words (the next layer's input).
//
// The reduction orders are those of the one-launch-per-step kernels (router
// kernel, bulk-copy gate/up kernel, down kernel, in either format), so the
// results are bit-identical to running the layers one by one.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "down.cuh"

namespace moe {

namespace {

constexpr int kSWarps = kStackThreads / 32;   // 24
constexpr int kSRouteWarps = kRouteThreads / 32;
constexpr size_t kStackSmemMax = 220 * 1024;  // dynamic; static shared memory is ~1.3 KB

static_assert(kStackThreads % 32 == 0 && kSWarps >= kSRouteWarps, "whole warps, router warps included");

// Word w of a spread exchange buffer (one 4-word piece per 128-byte line).
__device__ __forceinline__ uint2 *stk_word(uint2 *base, int w) {
    return base + (size_t)(w >> 2) * kStkLineWords + (w & 3);
}

// Tag of step l of a launch: 26 bits of launch count, 6 bits of layer.
__device__ __forceinline__ unsigned stk_tag(unsigned base, int l) {
    return (base << 6) | (unsigned)l;
}

constexpr int kAbortEvery = 256;   // polling rounds between two looks at the abort word
#ifndef MOE_STACK_POLL_SLEEP
#define MOE_STACK_POLL_SLEEP 16
#endif
constexpr int kPollSleepNs = MOE_STACK_POLL_SLEEP;  // back-off between polling rounds (ns)
constexpr int kXThreads = 256;     // threads that gather the layer input (one piece each at H = 2048)
constexpr int kHThreads = 256;     // threads that gather h
#ifndef MOE_STACK_PIECES
#define MOE_STACK_PIECES 4
#endif
constexpr int kStackPieces = MOE_STACK_PIECES;  // gate/up code pieces per CTA, landing in order
constexpr int kPollMaxJ = 4;       // pieces per polling thread

__device__ __forceinline__ uint64_t stk_clock() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// By the calling thread t of nt polling threads: the 32-byte pieces
// i = t, t + nt, ... < n of src (piece i = tagged words 4i .. 4i+3, at the
// start of line i of the spread layout; two single-copy-atomic 8-byte words
// per 16-byte load) until all four words of a
// piece carry `tag`; put(i, values) receives each piece as it lands.  Every
// round issues the loads of all pieces still missing at once, then checks
// them; between rounds the thread sleeps, and every kAbortEvery rounds it
// looks at the abort word (few threads poll, and rarely look there, so the
// polling does not crowd L2).  False on timeout or abort.
template <class Put>
__device__ __forceinline__ bool poll_pieces(const uint2 *src, int n, int t, int nt, unsigned tag,
                                            int limit, const unsigned *abort, unsigned base,
                                            Put &&put) {
    unsigned todo = 0;
#pragma unroll
    for (int j = 0; j < kPollMaxJ; ++j)
        if (t + j * nt < n) todo |= 1u << j;
    #pragma unroll 1
    for (int r = 0; todo && r < limit; ++r) {
        uint2 w[kPollMaxJ][4];
#pragma unroll
        for (int j = 0; j < kPollMaxJ; ++j)
            if ((todo >> j) & 1u) {
                const uint2 *q = src + (size_t)(t + j * nt) * kStkLineWords;
                ld_relaxed_gpu_2x64(q, w[j][0], w[j][1]);
                ld_relaxed_gpu_2x64(q + 2, w[j][2], w[j][3]);
            }
#pragma unroll
        for (int j = 0; j < kPollMaxJ; ++j)
            if (((todo >> j) & 1u) && w[j][0].x == tag && w[j][1].x == tag && w[j][2].x == tag &&
                w[j][3].x == tag) {
                put(t + j * nt, make_uint4(w[j][0].y, w[j][1].y, w[j][2].y, w[j][3].y));
                todo &= ~(1u << j);
            }
        if (!todo) break;
        if (r % kAbortEvery == kAbortEvery - 1 && ld_relaxed_gpu(abort) == base) return false;
        __nanosleep(kPollSleepNs);
    }
    return todo == 0;
}

// The layer input: pieces of x_tag -> sx (8 BF16 values per piece).  Out of
// line, so the polling registers do not add to the GEMV loops'.
static __device__ __noinline__ bool stk_gather_x(const uint2 *x_tag, int n, int t, unsigned tag,
                                                 int limit, const unsigned *abort, unsigned base,
                                                 uint4 *sx) {
    return poll_pieces(x_tag, n, t, kXThreads, tag, limit, abort, base,
                       [&](int i, uint4 v) { sx[i] = v; });
}

// All of h: pieces of h_tag -> the staged layout in shared memory (raw BF16,
// converted after the barrier), and each vector's max |h| into s_hmax.  Out of
// line.
static __device__ __noinline__ bool stk_gather_h(const uint2 *h_tag, int total, int npc, int t,
                                                 unsigned tag, int limit, const unsigned *abort,
                                                 unsigned base, uint4 *sv, unsigned *s_hmax) {
    return poll_pieces(h_tag, total, t, kHThreads, tag, limit, abort, base, [&](int i, uint4 v) {
        const int q = i / npc;
        const int pi = i - q * npc;
        sv[q * npc + h_piece(pi >> 2, pi & 3)] = v;
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        float m = 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r)
            m = fmaxf(m, fmaxf(fabsf(bf16_to_f32(w4[r] & 0xFFFFu)), fabsf(bf16_to_f32(w4[r] >> 16))));
        atomicMax(s_hmax + q, __float_as_uint(m));
    });
}

// By one warp: all n (<= 256) tagged logits (logit e on line e), copied into
// s_logits, with the same round structure.  Every lane returns the same
// verdict.  Out of line.
static __device__ __noinline__ bool stk_gather_logits(const uint2 *ent, int n, unsigned tag,
                                                      float *s_logits, int limit,
                                                      const unsigned *abort, unsigned base) {
    const int lane = threadIdx.x & 31;
    unsigned todo = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (lane + 32 * j < n) todo |= 1u << j;
    #pragma unroll 1
    for (int r = 0; r < limit; ++r) {
        uint2 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if ((todo >> j) & 1u)
                v[j] = ld_relaxed_gpu_v2(ent + (size_t)(lane + 32 * j) * kStkLineWords);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (((todo >> j) & 1u) && v[j].x == tag) {
                s_logits[lane + 32 * j] = __uint_as_float(v[j].y);
                todo &= ~(1u << j);
            }
        if (__all_sync(0xffffffffu, todo == 0)) {
            __syncwarp();
            return true;
        }
        if (r % kAbortEvery == kAbortEvery - 1 &&
            __shfl_sync(0xffffffffu, lane == 0 ? (int)(ld_relaxed_gpu(abort) == base) : 0, 0))
            return false;
        __nanosleep(kPollSleepNs);
    }
    return false;
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

// By one thread: every copy of the layer into shared memory, in the order the
// CTA needs the bytes -- the gate/up scales (on *sbar), the gate/up code rows
// in pieces of ppc row pairs (piece c on gbar[c]), then the down rows (on
// *dbar).  Bulk copies issued one after another by one thread land in that
// order at full bandwidth (issued together, they would share the memory
// system and all land at the end), so the GEMVs of the first pieces run while
// the later ones stream.  Gate/up layout: codes [2][NR][H/2] (gate, up), then
// scales [2][NR][H/32] (NVFP4: [2][NR][H/16]); down layout: codes [k][R][I/2],
// scales [k][R][I/32] (NVFP4: I/16).
// Out of line.
static __device__ __noinline__ void stk_issue_layer(
    const uint8_t *cb, const uint8_t *sb, const ExpertPtrs *tab, size_t cstride, size_t sstride,
    const int *s_ids, int E, int H, int I, int k, int pb0, int np, int ppc, int NR, uint8_t *gu,
    uint64_t *sbar, uint64_t *gbar, int r0, int r1, int R, uint8_t *rows_c, uint8_t *rows_s,
    uint64_t *dbar, uint64_t pol, int nv) {
    const size_t rc = (size_t)H >> 1, rs = (size_t)H >> (nv ? 4 : 5);
    auto codes = [&](int e, int m) {
        return cb ? cb + (size_t)(3 * e + m) * cstride : tab[e].codes[m];
    };
    auto scales = [&](int e, int m) {
        return cb ? sb + (size_t)(3 * e + m) * sstride : tab[e].scales[m];
    };
    // rows [g0, g1) of the flattened (slot, row) space, split by slot: f(q, e,
    // first row a, count n, local row lr, matrix row i0) for every valid slot
    auto segments = [&](int g0, int g1, auto &&f) {
        #pragma unroll 1
        for (int q = g0 / I; g1 > g0 && q <= (g1 - 1) / I; ++q) {
            const int e = s_ids[q];
            if (e < 0 || e >= E) continue;
            const int a = max(g0, q * I);
            const int n = min(g1, (q + 1) * I) - a;
            f(e, (size_t)n, (size_t)(a - 2 * pb0), (size_t)(a - q * I));
        }
    };
    const int g0 = 2 * pb0, g1 = 2 * (pb0 + np);
    unsigned bytes = 0;
    segments(g0, g1, [&](int, size_t n, size_t, size_t) { bytes += (unsigned)(2 * n * rs); });
    mbar_arrive_expect_tx(sbar, bytes);
    segments(g0, g1, [&](int e, size_t n, size_t lr, size_t i0) {
        #pragma unroll 1
        for (int m = 0; m < 2; ++m)
            bulk_g2s_hint(gu + 2 * (size_t)NR * rc + ((size_t)m * NR + lr) * rs, scales(e, m) + i0 * rs,
                          (unsigned)(n * rs), sbar, pol);
    });
    const int nch = (np + ppc - 1) / ppc;
    #pragma unroll 1
    for (int c = 0; c < nch; ++c) {
        const int a0 = 2 * (pb0 + c * ppc), a1 = 2 * (pb0 + min(np, (c + 1) * ppc));
        bytes = 0;
        segments(a0, a1, [&](int, size_t n, size_t, size_t) { bytes += (unsigned)(2 * n * rc); });
        mbar_arrive_expect_tx(&gbar[c], bytes);
        segments(a0, a1, [&](int e, size_t n, size_t lr, size_t i0) {
            #pragma unroll 1
            for (int m = 0; m < 2; ++m)
                bulk_g2s_hint(gu + ((size_t)m * NR + lr) * rc, codes(e, m) + i0 * rc,
                              (unsigned)(n * rc), &gbar[c], pol);
        });
    }
    const size_t drc = (size_t)I >> 1, drs = (size_t)I >> (nv ? 4 : 5), dn = (size_t)(r1 - r0);
    bytes = 0;
    #pragma unroll 1
    for (int j = 0; j < k; ++j) {
        const int e = s_ids[j];
        if (e >= 0 && e < E) bytes += (unsigned)(dn * (drc + drs));
    }
    mbar_arrive_expect_tx(dbar, bytes);
    #pragma unroll 1
    for (int j = 0; j < k && dn > 0; ++j) {
        const int e = s_ids[j];
        if (e < 0 || e >= E) continue;
        bulk_g2s_hint(rows_c + (size_t)j * R * drc, codes(e, 2) + (size_t)r0 * drc,
                      (unsigned)(dn * drc), dbar, pol);
        bulk_g2s_hint(rows_s + (size_t)j * R * drs, scales(e, 2) + (size_t)r0 * drs,
                      (unsigned)(dn * drs), dbar, pol);
    }
}

// Phase F: the down GEMV of the CTA's nr output rows for every slot, rows
// (codes [k][R][I/2], scales [k][R][I/32]) and the FP16-staged h ([k][I/2]
// words, h_piece order) in shared memory.  Warp w serves slot j = w % k; its
// teams of TLD lanes take local rows ti, ti + tps, ... two at a time (the
// h chunk loaded once for both rows), lane lt the 16-byte chunks lt + TLD u
// of each row, one E8M0 group each (NV: two E4M3 scales per chunk, each
// 16-element half sum scaled in FP32).  Per row the sums and their order are
// those of the per-layer down kernel (same bits).  so[j R + row] = BF16(o),
// o = sum * s_xs[j] (NV: s_xs holds the staging scale times the expert's down
// multiplier).
template <int TLD, int KCHD, bool NV>
__device__ __forceinline__ void stk_down_rows(int I, int k, int E, int R, int nr, const int *s_ids,
                                              const uint8_t *rows_c, const uint8_t *rows_s,
                                              const uint32_t *sh, const float *s_xs, float *so,
                                              unsigned *status) {
    constexpr int TPW = 32 / TLD;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int groups = kSWarps / k;  // warps per slot
    const int j = warp % k, gi = warp / k;
    if (gi >= groups) return;
    const int tps = groups * TPW;  // teams per slot
    const int lt = lane & (TLD - 1);
    const unsigned mask = team_mask<TLD>(lane);
    const int C = I >> 5;
    const size_t rc = (size_t)I >> 1, rs = (size_t)I >> (NV ? 4 : 5);
    const int e = s_ids[j];
    const bool bad = e < 0 || e >= E;
    const uint32_t *xv = sh + (size_t)j * (I >> 1);
    const float xs = s_xs[j];
    #pragma unroll 1
    for (int ra = gi * TPW + lane / TLD; ra < nr; ra += 2 * tps) {
        const int rb = ra + tps;
        const bool has_b = rb < nr;
        const uint8_t *ca = rows_c + (size_t)(j * R + ra) * rc, *sa = rows_s + (size_t)(j * R + ra) * rs;
        const uint8_t *cb = rows_c + (size_t)(j * R + rb) * rc, *sb = rows_s + (size_t)(j * R + rb) * rs;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int u = 0; u < KCHD; ++u) {
            const int c = lt + TLD * u;
            if (c < C && !bad) {
                const uint4 *xq = reinterpret_cast<const uint4 *>(xv + (size_t)c * 16);
                uint32_t x[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 v = xq[q ^ ((c >> 1) & 3)];  // h_piece order
                    x[4 * q] = v.x;
                    x[4 * q + 1] = v.y;
                    x[4 * q + 2] = v.z;
                    x[4 * q + 3] = v.w;
                }
                if (NV) {
                    float lo, hi, slo, shi;
                    dot32_e2m1_f16_halves(*reinterpret_cast<const uint4 *>(ca + (size_t)c * 16), x, lo,
                                          hi);
                    e4m3x2_to_f32(*reinterpret_cast<const uint16_t *>(sa + 2 * c), slo, shi);
                    a0 = fmaf(hi, shi, fmaf(lo, slo, a0));
                    if (has_b) {
                        dot32_e2m1_f16_halves(*reinterpret_cast<const uint4 *>(cb + (size_t)c * 16), x,
                                              lo, hi);
                        e4m3x2_to_f32(*reinterpret_cast<const uint16_t *>(sb + 2 * c), slo, shi);
                        a1 = fmaf(hi, shi, fmaf(lo, slo, a1));
                    }
                } else {
                    a0 = fmaf(dot32_e2m1_f16(*reinterpret_cast<const uint4 *>(ca + (size_t)c * 16), x),
                              e8m0_to_f32(sa[c]), a0);
                    if (has_b)
                        a1 = fmaf(
                            dot32_e2m1_f16(*reinterpret_cast<const uint4 *>(cb + (size_t)c * 16), x),
                            e8m0_to_f32(sb[c]), a1);
                }
            }
        }
        a0 = team_add<TLD>(a0, mask);
        a1 = team_add<TLD>(a1, mask);
        if (lt == 0) {
            so[j * R + ra] = bad ? 0.f : round_bf16(a0 * xs);
            if (has_b) so[j * R + rb] = bad ? 0.f : round_bf16(a1 * xs);
            if (bad) atomicOr(status, kBadExpertId);
        }
    }
}

}  // namespace

// Phase time stamps (profiling): thread 0 (or the producer's lane 0) of every
// CTA records the global timer at fixed points of each layer when p.trace is
// given: [L][grid][kStackTraceSlots].
#define STK_STAMP(slot)                                                                  \
    do {                                                                                 \
        if (p.trace && (tid == 0 || ((slot) == 3 || (slot) == 4 || (slot) >= 10)))       \
            p.trace[((size_t)l * G + b) * kStackTraceSlots + (slot)] = stk_clock();      \
    } while (0)

// KCH: 16-byte chunks per lane of a gate/up row (H = 32 * 32 * KCH at most);
// TLD / KCHD: the down phase's team of TLD lanes holding KCHD chunks each.
// NV: NVFP4 layers (E4M3 scale per 16 elements, FP32 multipliers per expert).
template <int KCH, int TLD, int KCHD, bool NV>
__global__ void __launch_bounds__(kStackThreads, 1)
stack_decode_kernel(const __grid_constant__ StackParams p) {
    extern __shared__ __align__(128) uint8_t sm[];
    __shared__ __align__(8) uint64_t sbar;                // gate/up scales
    __shared__ __align__(8) uint64_t gbar[kStackPieces];  // gate/up code pieces
    __shared__ __align__(8) uint64_t dbar;                // down rows
    __shared__ __align__(8) uint64_t rbar[2];             // router rows (next layer ahead)
    __shared__ int s_ids[kMaxTopK];
    __shared__ float s_w[kMaxTopK];
    __shared__ float s_logits[kFusedMaxE];
    __shared__ float s_red[3][kSRouteWarps];
    __shared__ float s_xs[kMaxTopK];
    __shared__ unsigned s_hmax[kMaxTopK];
    __shared__ unsigned s_base;
    __shared__ int s_x16exp;
    __shared__ int s_fail;
    __shared__ int s_copied;                // layer whose weight copies were issued
    __shared__ int s_rt_armed[2];           // layer whose router row went into buffer i
    __shared__ StackLayer s_layers[kStackMaxLayers];  // the layer table, read once per launch
    __shared__ float s_bias[kStackMaxLayers];         // router bias of expert b, every layer

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = (int)blockIdx.x, G = (int)gridDim.x;
    const int E = p.E, H = p.H, I = p.I, k = p.k, L = p.L;
    const int nch8 = H >> 3;  // 16-byte pieces of a BF16 vector
    const int limit = p.spin_limit;
    // this CTA's shares: gate/up row pairs [pb0, pb0 + np), down rows [r0, r1)
    const int P = k * I / 2;
    const int pb0 = (int)((long long)P * b / G);
    const int np = (int)((long long)P * (b + 1) / G) - pb0;
    const int NU = H / p.plan.U;
    const int r0 = p.plan.U * (int)((long long)NU * b / G);
    const int r1 = p.plan.U * (int)((long long)NU * (b + 1) / G);
    uint16_t *rbuf = reinterpret_cast<uint16_t *>(sm + p.plan.off_rt);  // [2][H]
    uint32_t *sx = reinterpret_cast<uint32_t *>(sm + p.plan.off_sx);    // [H/2] layer input

    if (tid == 0) {
        mbar_init(&sbar, 1);
        #pragma unroll 1
        for (int c = 0; c < kStackPieces; ++c) mbar_init(&gbar[c], 1);
        mbar_init(&dbar, 1);
        mbar_init(&rbar[0], 1);
        mbar_init(&rbar[1], 1);
        mbar_fence_init();
        // launches made so far by CTA b (every launch runs every CTA, so all
        // CTAs agree); written by the previous launch, complete before this one
        s_base = ld_relaxed_gpu(p.seq + b) + 1u;
        s_fail = 0;
        s_copied = -1;
        s_rt_armed[0] = s_rt_armed[1] = -1;
    }
    // the layer table into shared memory (kernel parameters indexed by layer
    // would be a constant-cache miss per layer), and this CTA's router bias of
    // every layer (loaded in parallel now, off the per-layer critical path)
    if (tid < L) {
        s_layers[tid] = p.layer[tid];
        const float *bias = p.layer[tid].bias;
        s_bias[tid] = (bias && b < E) ? bias[b] : 0.f;
    }
    __syncthreads();
    const unsigned base = s_base;
    if (warp == kSWarps - 1 && lane == 0 && b < E) {
        stk_issue_router(s_layers[0].router_w, b, H, rbuf, &rbar[0]);
        s_rt_armed[0] = 0;
    }

    int l = 0;
    #pragma unroll 1
    for (; l < L; ++l) {
        const unsigned tag = stk_tag(base, l);
        const StackLayer &ly = s_layers[l];
        STK_STAMP(0);

        // ---- A: layer input r -> sx ----
        bool ok = true;
        if (l == 0) {
            const uint32_t *r32 = reinterpret_cast<const uint32_t *>(p.r);
            #pragma unroll 1
            for (int m = tid; m < (H >> 1); m += kStackThreads) sx[m] = r32[m];
        } else if (tid < kXThreads) {
            // the previous layer's tagged outputs, 8 values per piece
            ok = stk_gather_x(p.x_tag, H >> 3, tid, tag - 1u, limit, p.abort, base,
                              reinterpret_cast<uint4 *>(sx));
        }
        if (!__syncthreads_and(ok)) break;
        STK_STAMP(1);
        if (b == 0 && p.r_hist) {
            uint32_t *dst = reinterpret_cast<uint32_t *>(p.r_hist + (size_t)l * H);
            #pragma unroll 1
            for (int m = tid; m < (H >> 1); m += kStackThreads) dst[m] = sx[m];
        }

        // ---- A: RMSNorm, router logit b, FP16 staging (threads of warps 0..7,
        // in the reduction order of the standalone router kernel) ----
        if (tid < kRouteThreads) {
            uint32_t *sx16 = reinterpret_cast<uint32_t *>(sm + p.plan.off_x16);
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
            float acc = 0.f, amax = 0.f;
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
                if (ly.bias) logit += s_bias[l];
                st_relaxed_gpu_v2(p.lg_tag + (size_t)b * kStkLineWords, tag,
                                  __float_as_uint(logit));
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
        STK_STAMP(2);

        // ---- C: routing (the last warp), then every copy of the layer (all) ----
        if (warp == kSWarps - 1) {
            const bool got = stk_gather_logits(p.lg_tag, E, tag, s_logits, limit, p.abort, base);
            if (got) {
                if (lane == 0) STK_STAMP(3);
                int id;
                float w;
                warp_topk_any<true>(s_logits, E, k, lane, id, w);
                if (lane < k) {
                    s_ids[lane] = id;
                    s_w[lane] = w;
                    if (b == 0 && p.ids_hist) p.ids_hist[(size_t)l * k + lane] = id;
                    if (b == 0 && p.w_hist) p.w_hist[(size_t)l * k + lane] = w;
                }
                if (lane == 0) STK_STAMP(10);
                if (lane == 1 && b < E && l + 1 < L) {
                    const int nb = (l + 1) & 1;
                    stk_issue_router(s_layers[l + 1].router_w, b, H, rbuf + (size_t)nb * H,
                                     &rbar[nb]);
                    s_rt_armed[nb] = l + 1;
                }
            } else if (lane == 0) {
                s_fail = 1;
            }
        }
        __syncthreads();
        if (s_fail) break;
        const int ppc = p.plan.ppc;
        const int NR = 2 * p.plan.np_max;
        uint8_t *gu = sm + p.plan.off_gu;
        if (tid == kStackThreads - 32) {
            // the producer warp's lane 0: every copy of the layer, in order
            uint8_t *rows_c = sm + p.plan.off_dn;
            stk_issue_layer(ly.codes_base, ly.scales_base, ly.table, p.codes_stride, p.scales_stride,
                            s_ids, E, H, I, k, pb0, np, ppc, NR, gu, &sbar, gbar, r0, r1, p.plan.R,
                            rows_c, rows_c + (size_t)k * p.plan.R * ((size_t)I >> 1), &dbar,
                            l2_evict_first_policy(), NV ? 1 : 0);
            s_copied = l;
            STK_STAMP(4);
        }

        // ---- D: gate/up + SwiGLU, one row pair per warp per step, each as
        // its code piece lands.  Lane l holds the 16-byte chunks l + 32 u
        // (u < KCH) of each row, one E8M0 group each; sums in the order of the
        // bulk-copy gate/up kernel. ----
        {
            const float xs = pow2(s_x16exp);
            const uint4 *sx16 = reinterpret_cast<const uint4 *>(sm + p.plan.off_x16);
            const int C = H >> 5;
            const size_t rc = (size_t)H >> 1, rs = (size_t)H >> (NV ? 4 : 5);
            if (warp < np && !mbar_wait(&sbar, (unsigned)l & 1u)) ok = false;
            #pragma unroll 1
            for (int pp = warp; pp < np && ok; pp += kSWarps) {
                if (!mbar_wait(&gbar[pp / ppc], (unsigned)l & 1u)) {
                    ok = false;
                    break;
                }
                if (tid == 0 && pp == 0) STK_STAMP(9);
                const int gr = 2 * (pb0 + pp);  // global row of the pair's first row
                const int e = s_ids[gr / I];
                const bool bad = e < 0 || e >= E;
                const size_t lr = (size_t)(2 * pp);
                float v[2][2];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                    for (int m = 0; m < 2; ++m) v[rr][m] = 0.f;
#pragma unroll
                for (int u = 0; u < KCH; ++u) {
                    const int c = lane + 32 * u;
                    uint4 cw[2][2];
                    uint32_t sw[2][2];
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            const size_t row = (size_t)m * NR + lr + rr;
                            if (c < C && !bad) {
                                cw[rr][m] = *reinterpret_cast<const uint4 *>(gu + row * rc + (size_t)c * 16);
                                sw[rr][m] = NV ? *reinterpret_cast<const uint16_t *>(
                                                     gu + 2 * (size_t)NR * rc + row * rs + 2 * c)
                                               : gu[2 * (size_t)NR * rc + row * rs + c];
                            } else {
                                cw[rr][m] = make_uint4(0u, 0u, 0u, 0u);
                                sw[rr][m] = NV ? 0x3838u : 127u;
                            }
                        }
                    if (NV) {
                        // each chunk's two 16-element halves (words 0-1, 2-3),
                        // each half sum scaled by its E4M3 scale in FP32 (the
                        // order of chunks_dot_nv)
                        float a[2][2][4];
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                            for (int m = 0; m < 2; ++m)
#pragma unroll
                                for (int i = 0; i < 4; ++i) a[rr][m][i] = 0.f;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint4 xv = c < C ? sx16[c * 4 + q4] : make_uint4(0u, 0u, 0u, 0u);
                            const int i0 = (q4 & 1) * 2;
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                                for (int m = 0; m < 2; ++m) {
                                    const uint4 cc = cw[rr][m];
                                    const uint32_t w = q4 == 0 ? cc.x : q4 == 1 ? cc.y : q4 == 2 ? cc.z : cc.w;
                                    dot8_e2m1_f16(w, xv.x, xv.y, xv.z, xv.w, a[rr][m][i0], a[rr][m][i0 + 1]);
                                }
                            if (q4 & 1) {
#pragma unroll
                                for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                                    for (int m = 0; m < 2; ++m) {
                                        float slo, shi;
                                        e4m3x2_to_f32(sw[rr][m], slo, shi);
                                        const float half = (a[rr][m][0] + a[rr][m][1]) + (a[rr][m][2] + a[rr][m][3]);
                                        v[rr][m] = fmaf(half, q4 == 1 ? slo : shi, v[rr][m]);
#pragma unroll
                                        for (int i = 0; i < 4; ++i) a[rr][m][i] = 0.f;
                                    }
                            }
                        }
                    } else {
                        float a[2][2][2];  // [row][gate, up][even, odd elements]
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                            for (int m = 0; m < 2; ++m) a[rr][m][0] = a[rr][m][1] = 0.f;
                        // the chunk's four 8-element pieces in order, each against
                        // all four rows (per row the order of chunks_dot)
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const uint4 xv = c < C ? sx16[c * 4 + q4] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                                for (int m = 0; m < 2; ++m) {
                                    const uint4 cc = cw[rr][m];
                                    const uint32_t w = q4 == 0 ? cc.x : q4 == 1 ? cc.y : q4 == 2 ? cc.z : cc.w;
                                    dot8_e2m1_f16(w, xv.x, xv.y, xv.z, xv.w, a[rr][m][0], a[rr][m][1]);
                                }
                        }
#pragma unroll
                        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                            for (int m = 0; m < 2; ++m)
                                v[rr][m] = fmaf(a[rr][m][0] + a[rr][m][1], e8m0_to_f32(sw[rr][m]), v[rr][m]);
                    }
                }
#pragma unroll
                for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                    for (int m = 0; m < 2; ++m) v[rr][m] = warp_sum(v[rr][m]);
                if (tid == 0 && pp == 0) STK_STAMP(11);
                if (lane == 0) {
                    uint32_t word = 0u;
                    // NVFP4: the expert's gate/up multiplier joins the exact
                    // power-of-two staging scale (as in the per-layer kernel)
                    const float sx = NV && !bad ? xs * __ldg(ly.gscale + 2 * e) : xs;
                    if (!bad)
                        word = (uint32_t)f32_to_bf16(swiglu_h(v[0][0], v[0][1], sx)) |
                               ((uint32_t)f32_to_bf16(swiglu_h(v[1][0], v[1][1], sx)) << 16);
                    else
                        atomicOr(p.status, kBadExpertId);
                    st_relaxed_gpu_v2(stk_word(p.h_tag, gr / 2), tag, word);
                }
            }
        }
        if (tid < k) s_hmax[tid] = 0u;
        if (!__syncthreads_and(ok)) break;
        STK_STAMP(5);

        // ---- E: all of h (tagged) -> FP16 in shared memory ----
        const int npc = I >> 3;  // 8-element pieces per vector
        const int total = k * npc;
        uint4 *sv = reinterpret_cast<uint4 *>(sm + p.plan.off_sh);
        if (tid < kHThreads)
            ok = stk_gather_h(p.h_tag, total, npc, tid, tag, limit, p.abort, base, sv, s_hmax);
        // the CTA's down rows (requested with the gate/up rows) must have landed
        if (tid == 0 && !mbar_wait(&dbar, (unsigned)l & 1u)) ok = false;
        if (!__syncthreads_and(ok)) break;
        STK_STAMP(6);
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
        if (tid < k) {
            const float xs = pow2(f16_stage_exponent(__uint_as_float(s_hmax[tid])));
            const int e = s_ids[tid];
            // NVFP4: times the expert's down multiplier (an exact product)
            s_xs[tid] = NV && e >= 0 && e < E ? xs * __ldg(ly.gscale + 2 * e + 1) : xs;
        }
        __syncthreads();
        STK_STAMP(15);

        // ---- F: down GEMV of the CTA's output rows, every slot ----
        const int R = p.plan.R;
        float *so = reinterpret_cast<float *>(sm + p.plan.off_so);  // [k][R] expert outputs
        if (r0 < r1) {
            const uint8_t *rows_c = sm + p.plan.off_dn;
            stk_down_rows<TLD, KCHD, NV>(I, k, E, R, r1 - r0, s_ids, rows_c,
                                     rows_c + (size_t)k * R * ((size_t)I >> 1),
                                     reinterpret_cast<const uint32_t *>(sv), s_xs, so, p.status);
        }
        __syncthreads();
        STK_STAMP(7);

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
            st_relaxed_gpu_v2(stk_word(p.x_tag, n / 2), tag, word);
            if (l == L - 1) reinterpret_cast<uint32_t *>(p.r)[n / 2] = word;
        }
        __syncthreads();  // sx, so, s_w are rewritten by the next layer
        STK_STAMP(8);
    }

    if (l < L) {
        // gave up: record it, release the other CTAs, and let no copy of this
        // CTA outlive it (the layer's copies and the router rows in flight;
        // waits bounded, a completed wait returns at once)
        if (tid == 0) {
            atomicOr(p.status, kTimeoutStatus);
            st_relaxed_gpu(p.abort, base);
            if (s_copied == l) {
                const int nch = (np + p.plan.ppc - 1) / p.plan.ppc;
                mbar_wait(&sbar, (unsigned)l & 1u);
                for (int c = 0; c < nch; ++c) mbar_wait(&gbar[c], (unsigned)l & 1u);
                mbar_wait(&dbar, (unsigned)l & 1u);
            }
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

template <int KCH, int TLD, int KCHD, bool NV>
cudaError_t launch_stk(const StackParams &p, int grid, cudaStream_t s) {
    static PerDeviceOnce once;
    cudaError_t e = per_device_once(once, [] {
        return cudaFuncSetAttribute(stack_decode_kernel<KCH, TLD, KCHD, NV>,
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
    return cudaLaunchKernelEx(&cfg, stack_decode_kernel<KCH, TLD, KCHD, NV>, p);
}

size_t al128(size_t v) { return (v + 127) & ~(size_t)127; }

}  // namespace

bool stack_plan(int E, int H, int I, int k, int grid, StackPlan *pl, int nv) {
    if (grid < 1 || E < 1 || E > grid || E > kFusedMaxE || k < 1 || k > kMaxTopK || k > E)
        return false;
    if (H % 512 != 0 || H > 2048 || I % 128 != 0 || I > 4096) return false;
    if (stack_variant(H, I) < 0) return false;
    // the gathering threads hold at most kPollMaxJ pieces each
    if (H / 8 > kXThreads * kPollMaxJ || k * I / 8 > kHThreads * kPollMaxJ) return false;
    StackPlan s = {};
    // rows per unit (even: the combine writes row pairs): U * (I/32 or I/16)
    // scale bytes are a 16-byte multiple
    s.U = nv ? 2 : ((I % 256 == 0) ? 2 : 4);
    const int NU = H / s.U;
    s.R = s.U * ((NU + grid - 1) / grid);
    if (kSWarps / k < 1) return false;  // the down phase needs a warp per slot
    const int P = k * I / 2;
    s.np_max = (P + grid - 1) / grid;
    s.ppc = (s.np_max + kStackPieces - 1) / kStackPieces;
    const size_t rc = (size_t)H / 2, rs = (size_t)H / (nv ? 16 : 32);
    size_t off = 0;
    s.off_gu = (unsigned)off;
    off = al128(off + (size_t)2 * s.np_max * 2 * (rc + rs));
    s.off_dn = (unsigned)off;
    off = al128(off + (size_t)k * s.R * ((size_t)I / 2 + (size_t)I / (nv ? 16 : 32)));
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
    const bool nv = p.nv != 0;
    switch (stack_variant(p.H, p.I)) {
    case 0: return nv ? launch_stk<1, 4, 3, true>(p, grid, s) : launch_stk<1, 4, 3, false>(p, grid, s);
    case 1: return nv ? launch_stk<1, 16, 1, true>(p, grid, s) : launch_stk<1, 16, 1, false>(p, grid, s);
    case 2: return nv ? launch_stk<1, 32, 1, true>(p, grid, s) : launch_stk<1, 32, 1, false>(p, grid, s);
    case 3: return nv ? launch_stk<2, 16, 3, true>(p, grid, s) : launch_stk<2, 16, 3, false>(p, grid, s);
    case 4: return nv ? launch_stk<2, 32, 2, true>(p, grid, s) : launch_stk<2, 32, 2, false>(p, grid, s);
    case 5: return nv ? launch_stk<2, 16, 1, true>(p, grid, s) : launch_stk<2, 16, 1, false>(p, grid, s);
    case 6: return nv ? launch_stk<2, 32, 1, true>(p, grid, s) : launch_stk<2, 32, 1, false>(p, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
