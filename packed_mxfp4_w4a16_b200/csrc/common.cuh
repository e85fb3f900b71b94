// common.cuh — device helpers shared by the sm_100a kernels of this library.
//
// Number formats (model card "LFM2.5-24B-A2B — Packed MXFP4 Inference", table
// "Model and quantization"): weights are E2M1 FP4 codes, two per byte, each 32
// consecutive K elements share one E8M0 exponent; activations and outputs are
// BF16; dot products accumulate in FP32.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Addresses of one expert's three packed matrices (0 gate, 1 up, 2 down):
// codes [rows][K/2] and E8M0 scales [rows][K/32] of each.
struct ExpertPtrs {
    const uint8_t *codes[3];
    const uint8_t *scales[3];
};

// ----------------------------------------------------------------- BF16 --

__device__ __forceinline__ float bf16_to_f32(uint32_t b) {
    return __uint_as_float(b << 16);
}

// Round an FP32 value to BF16 (nearest, ties to even; NaN stays NaN).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

// Round to BF16 and back: the value of a BF16 rounding point.
__device__ __forceinline__ float round_bf16(float f) {
    return bf16_to_f32(f32_to_bf16(f));
}

// ------------------------------------------------------------ loads ------

// 16-byte streaming load of read-only data: no L1 allocation, 256-byte L2
// fetch granularity (the rows are streamed once per call).
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

// The same with an L2 eviction policy (createpolicy) for the source lines.
// Volatile: issued where written (a batch of these is meant to be in flight
// before the first result is used; a plain asm could be sunk to its use).
__device__ __forceinline__ uint4 ld_stream16_hint(const void *p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p), "l"(pol));
    return r;
}
__device__ __forceinline__ uint32_t ld_stream_u8_hint(const uint8_t *p, uint64_t pol) {
    uint16_t r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.u8 %0, [%1], %2;" : "=h"(r)
                 : "l"(p), "l"(pol));
    return r;
}

__device__ __forceinline__ uint32_t ld_stream_u8(const uint8_t *p) {
    uint16_t r;
    asm("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// Hint: bring [p, p + bytes) into L2 (bytes a multiple of 16, p 16-aligned).
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes)
                 : "memory");
}

// -------------------------------------------------------- E8M0 / E2M1 ----

// 2^(e-127) in FP32: e = 0 gives the subnormal 2^-127, e = 255 gives NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
    uint32_t bits = e << 23;
    bits = (e == 0u) ? 0x00400000u : bits;
    bits = (e == 255u) ? 0x7FC00000u : bits;
    return __uint_as_float(bits);
}

// The 16-entry E2M1 table applied in registers by the sm_100a conversion
// instruction: each byte of w (two codes, low nibble = lower element) becomes
// an f16x2 word, exactly (every E2M1 value is an FP16 value).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t (&out)[4]) {
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t"
        "}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
        : "r"(w));
}

// d = A B + c for one m16n8k16 tile, FP16 operands, FP32 accumulators.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1, const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

// One 32-element scale group of 16 packed rows against 8 FP16 columns on the
// tensor cores, scaled per row by the group's E8M0 exponent and added to acc.
// The group's K order is permuted identically for A and B: thread (g, q) of
// the warp supplies codes 8q..8q+7 of rows g and g+8 (one 4-byte word each,
// w_lo / w_hi) and elements 8q..8q+7 of column g (b).  Slots 2q, 2q+1 / 2q+8,
// 2q+9 of the first MMA then carry elements 8q + {0,1} / {2,3}, of the second
// 8q + {4,5} / {6,7}.  The group's partial product (fresh accumulator) times
// the row's 2^(e-127) is added in FP32: exactly per-group scaling.
// acc: rows g / g + 8 x columns 2q, 2q + 1 (acc[0], acc[1] / acc[2], acc[3]).
__device__ __forceinline__ void mma_group_e2m1(float (&acc)[4], uint32_t w_lo, uint32_t w_hi,
                                               uint32_t s_lo, uint32_t s_hi, const uint4 &b) {
    uint32_t fa[2][4];
    e2m1x8_to_f16x8(w_lo, fa[0]);
    e2m1x8_to_f16x8(w_hi, fa[1]);
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    float dd[4];
    mma_f16(dd, fa[0][0], fa[1][0], fa[0][1], fa[1][1], b.x, b.y, zero);
    mma_f16(dd, fa[0][2], fa[1][2], fa[0][3], fa[1][3], b.z, b.w, dd);
    const float sl = e8m0_to_f32(s_lo), sh = e8m0_to_f32(s_hi);
    acc[0] = fmaf(dd[0], sl, acc[0]);
    acc[1] = fmaf(dd[1], sl, acc[1]);
    acc[2] = fmaf(dd[2], sh, acc[2]);
    acc[3] = fmaf(dd[3], sh, acc[3]);
}

// NVFP4 form of the same: a 32-element group is two 16-element blocks with
// their own E4M3 scales (sc_lo: the two scale bytes of row g, block 0 in the
// low byte; sc_hi: those of row g + 8).  Thread (g, q) supplies codes
// 4q..4q+3 of block 0 in the low half of its word and codes 4q..4q+3 of block
// 1 in the high half (w_lo: row g, w_hi: row g + 8), and the activations of
// column g in the same order (b.x, b.y: block 0 elements 4q..4q+3; b.z, b.w:
// block 1).  The first MMA then sums block 0 and the second block 1, each
// from a fresh accumulator; each block's partial product times its row's
// E4M3 scale is added to acc in FP32, block 0 first: exactly per-block scaling.
__device__ __forceinline__ void mma_group_nvfp4(float (&acc)[4], uint32_t w_lo, uint32_t w_hi,
                                                uint32_t sc_lo, uint32_t sc_hi, const uint4 &b);

__device__ __forceinline__ float f16_bits_to_f32(uint32_t h) {
    float f;
    asm("{ .reg .f16 t; mov.b16 t, %1; cvt.f32.f16 %0, t; }" : "=f"(f) : "h"((uint16_t)h));
    return f;
}

// Dot product of 8 packed E2M1 codes (one 32-bit word, element order: byte 0
// low nibble first) with 8 FP16 activations (four f16x2 words), accumulated
// in FP32 (each product is exact, one rounding per add).  a0 receives the
// even elements, a1 the odd ones.
__device__ __forceinline__ void dot8_e2m1_f16(uint32_t w, uint32_t x01, uint32_t x23,
                                              uint32_t x45, uint32_t x67, float &a0,
                                              float &a1) {
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        ".reg .b32 p0, p1, p2, p3;\n\t"
        ".reg .f16 w0, w1, w2, w3, w4, w5, w6, w7;\n\t"
        ".reg .f16 x0, x1, x2, x3, x4, x5, x6, x7;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 p0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 p1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 p2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 p3, b3;\n\t"
        "mov.b32 {w0, w1}, p0;\n\t"
        "mov.b32 {w2, w3}, p1;\n\t"
        "mov.b32 {w4, w5}, p2;\n\t"
        "mov.b32 {w6, w7}, p3;\n\t"
        "mov.b32 {x0, x1}, %3;\n\t"
        "mov.b32 {x2, x3}, %4;\n\t"
        "mov.b32 {x4, x5}, %5;\n\t"
        "mov.b32 {x6, x7}, %6;\n\t"
        "fma.rn.f32.f16 %0, w0, x0, %0;\n\t"
        "fma.rn.f32.f16 %1, w1, x1, %1;\n\t"
        "fma.rn.f32.f16 %0, w2, x2, %0;\n\t"
        "fma.rn.f32.f16 %1, w3, x3, %1;\n\t"
        "fma.rn.f32.f16 %0, w4, x4, %0;\n\t"
        "fma.rn.f32.f16 %1, w5, x5, %1;\n\t"
        "fma.rn.f32.f16 %0, w6, x6, %0;\n\t"
        "fma.rn.f32.f16 %1, w7, x7, %1;\n\t"
        "}"
        : "+f"(a0), "+f"(a1)
        : "r"(w), "r"(x01), "r"(x23), "r"(x45), "r"(x67));
}

// One 32-element group (16 code bytes) against its 32 FP16 activations
// (16 f16x2 words): the unscaled partial sum of the group.
__device__ __forceinline__ float dot32_e2m1_f16(const uint4 &c, const uint32_t *x) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    dot8_e2m1_f16(c.x, x[0], x[1], x[2], x[3], a0, a1);
    dot8_e2m1_f16(c.y, x[4], x[5], x[6], x[7], a2, a3);
    dot8_e2m1_f16(c.z, x[8], x[9], x[10], x[11], a0, a1);
    dot8_e2m1_f16(c.w, x[12], x[13], x[14], x[15], a2, a3);
    return (a0 + a1) + (a2 + a3);
}

// NVFP4 ("primitive-ai/LFM2.5-24B-A2B-NVFP4A16", "What's quantized to
// what"): a 32-element chunk carries two 16-element blocks, each with its own
// FP8 E4M3 scale.  The two unscaled half sums of the chunk (codes 0..15 in
// c.x, c.y; 16..31 in c.z, c.w).
__device__ __forceinline__ void dot32_e2m1_f16_halves(const uint4 &c, const uint32_t *x,
                                                      float &lo, float &hi) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    dot8_e2m1_f16(c.x, x[0], x[1], x[2], x[3], a0, a1);
    dot8_e2m1_f16(c.y, x[4], x[5], x[6], x[7], a2, a3);
    lo = (a0 + a1) + (a2 + a3);
    a0 = a1 = a2 = a3 = 0.f;
    dot8_e2m1_f16(c.z, x[8], x[9], x[10], x[11], a0, a1);
    dot8_e2m1_f16(c.w, x[12], x[13], x[14], x[15], a2, a3);
    hi = (a0 + a1) + (a2 + a3);
}

// Two FP8 E4M3 scales (the low and high byte of s) as FP32, exactly: the
// sm_100a conversion instruction to f16x2 (every E4M3 value, subnormals and
// NaN included, is an FP16 value), then FP16 -> FP32.
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t s, float &lo, float &hi) {
    uint32_t h2;
    asm("{\n\t"
        ".reg .b16 t;\n\t"
        "cvt.u16.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, t;\n\t"
        "}"
        : "=r"(h2)
        : "r"(s));
    lo = f16_bits_to_f32(h2 & 0xFFFFu);
    hi = f16_bits_to_f32(h2 >> 16);
}

__device__ __forceinline__ void mma_group_nvfp4(float (&acc)[4], uint32_t w_lo, uint32_t w_hi,
                                                uint32_t sc_lo, uint32_t sc_hi, const uint4 &b) {
    uint32_t fa[2][4];
    e2m1x8_to_f16x8(w_lo, fa[0]);
    e2m1x8_to_f16x8(w_hi, fa[1]);
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    float d0[4], d1[4];
    mma_f16(d0, fa[0][0], fa[1][0], fa[0][1], fa[1][1], b.x, b.y, zero);
    mma_f16(d1, fa[0][2], fa[1][2], fa[0][3], fa[1][3], b.z, b.w, zero);
    float l0, l1, h0, h1;
    e4m3x2_to_f32(sc_lo, l0, l1);
    e4m3x2_to_f32(sc_hi, h0, h1);
    acc[0] = fmaf(d1[0], l1, fmaf(d0[0], l0, acc[0]));
    acc[1] = fmaf(d1[1], l1, fmaf(d0[1], l0, acc[1]));
    acc[2] = fmaf(d1[2], h1, fmaf(d0[2], h0, acc[2]));
    acc[3] = fmaf(d1[3], h1, fmaf(d0[3], h0, acc[3]));
}

// sym8 form (int8 weights, one binary16 scale per 32 K elements): thread
// (g, q) supplies weights 8q..8q+7 of rows g and g + 8 (8 bytes each, w_lo /
// w_hi) and elements 8q..8q+7 of column g (b), in the K order of
// mma_group_e2m1.  A weight byte q becomes FP16 exactly: its biased value
// q + 128 is the low mantissa byte of the FP16 1024 + (q + 128), and one
// subtraction of 1152 leaves q (an integer below 2^11).  The group's partial
// product (fresh accumulator, exact products) times the row's scale (s_lo /
// s_hi: binary16 bits, FP32 exactly) is added to acc in FP32.
__device__ __forceinline__ void s8x8_to_f16x8(uint2 w, uint32_t (&out)[4]) {
    const uint32_t u0 = w.x ^ 0x80808080u, u1 = w.y ^ 0x80808080u;
    const uint32_t hi = 0x64646464u;  // high byte of 1024 + b in FP16
    const uint32_t bias = 0x64806480u;  // 1152 in both halves
    const uint32_t p[4] = {__byte_perm(u0, hi, 0x5150u), __byte_perm(u0, hi, 0x5352u),
                           __byte_perm(u1, hi, 0x5150u), __byte_perm(u1, hi, 0x5352u)};
#pragma unroll
    for (int i = 0; i < 4; ++i) asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(out[i]) : "r"(p[i]), "r"(bias));
}

__device__ __forceinline__ void mma_group_s8(float (&acc)[4], uint2 w_lo, uint2 w_hi,
                                             uint32_t s_lo, uint32_t s_hi, const uint4 &b) {
    uint32_t fa[2][4];
    s8x8_to_f16x8(w_lo, fa[0]);
    s8x8_to_f16x8(w_hi, fa[1]);
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    float dd[4];
    mma_f16(dd, fa[0][0], fa[1][0], fa[0][1], fa[1][1], b.x, b.y, zero);
    mma_f16(dd, fa[0][2], fa[1][2], fa[0][3], fa[1][3], b.z, b.w, dd);
    const float sl = f16_bits_to_f32(s_lo), sh = f16_bits_to_f32(s_hi);
    acc[0] = fmaf(dd[0], sl, acc[0]);
    acc[1] = fmaf(dd[1], sl, acc[1]);
    acc[2] = fmaf(dd[2], sh, acc[2]);
    acc[3] = fmaf(dd[3], sh, acc[3]);
}

// ------------------------------------------------ FP16 staging of BF16 ----
// The GEMVs multiply FP16 weights (exact E2M1 values) with activations held
// in FP16.  A BF16 vector v is staged as v * 2^-c with c chosen from max|v|
// so that the largest element lands in [2^14, 2^15): every element within
// 2^29 of the maximum converts exactly (BF16 has 8 significant bits, FP16
// 11), smaller ones lose bits far below FP32 accumulation noise.  The dot
// product is multiplied back by 2^c in FP32.

__device__ __forceinline__ int f16_stage_exponent(float amax) {
    if (!(amax > 0.f) || !(amax <= 3.0e38f))
        return 0;  // zero, NaN or inf: stage unscaled
    int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
    // c = (biased exponent of max) - 127 - 14, clamped so that 2^-c stays a
    // normal FP32 value (vectors whose max is below 2^-113 are staged with
    // less headroom; they are far below any activation scale in practice)
    int c = e - 141;
    return c < -127 ? -127 : c;
}

// 2^-c for c in [-127, 113], exact, as an FP32 normal number.
__device__ __forceinline__ float pow2_neg(int c) {
    return __uint_as_float((uint32_t)(127 - c) << 23);
}

// 2^c for c in [-127, 113], exact (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2(int c) {
    return c >= -126 ? __uint_as_float((uint32_t)(c + 127) << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ uint16_t f32_to_f16_bits(float f) {
    uint16_t r;
    asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

// Two FP32 values -> one f16x2 word (lo in the low half), round to nearest.
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ------------------------------------------------- mbarrier / bulk copy ----
// Shared-memory barriers that count completed bytes of asynchronous bulk
// copies (TMA engine, non-tensor form: 16-byte aligned addresses, sizes in
// multiples of 16 bytes).  Every wait is bounded: after kMaxSpin unsuccessful
// polls it gives up and the caller records an error in the status word.

constexpr unsigned kTimeoutStatus = 0x2u;  // a bounded wait gave up
constexpr int kMaxSpin = 1 << 20;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// producer: announce `bytes` of incoming copies and arrive (count 1)
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; "
        "selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; false if it did not within
// kMaxSpin polls.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity) {
#pragma unroll 1
    for (int i = 0; i < kMaxSpin; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// L2 eviction priorities for cache-hinted accesses.  The packed expert rows
// are read once per token and stream through L2 far faster than it holds
// them (hundreds of MB per token against 126 MB): marked evict-first, they
// leave the small state that every layer reuses (router weights, activations,
// routing, kernel code) in L2.  The router weights are marked evict-last.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Global -> shared bulk copy completing `bytes` on `bar`, with an L2
// eviction policy for the source lines.
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, unsigned bytes,
                                              uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
        "[%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// 16-byte global load with an L2 eviction policy.
__device__ __forceinline__ uint4 ld_hint16(const void *p, uint64_t pol) {
    uint4 r;
    asm volatile("ld.global.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(pol));
    return r;
}

// ------------------------------------------------------------- warps -----

template <int TL>
__device__ __forceinline__ float team_sum(float v) {
#pragma unroll
    for (int o = TL / 2; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------- top-k --
// Top-k of one token's logits (E values in global memory, read through L2):
// descending, equal logits -> lower expert id, NaN never chosen; coefficients
// = softmax over the k chosen logits.  Called by one full warp; every lane
// returns the same ids[0..k) and w[0..k).  Each round takes the warp-wide max
// of an order-preserving key, then the lowest id among lanes holding it.
__device__ __forceinline__ uint32_t logit_key(float v) {
    const uint32_t b = __float_as_uint(v);
    return (v != v) ? 0u : ((b & 0x80000000u) ? ~b : (b | 0x80000000u));
}

// Top-k of one token's E logits by one warp (strictly greater wins, the lower
// expert id on equal keys), then the coefficients.  Lane j (j < k) returns
// the j-th selection in (id, w); other lanes return id = -1.  Round j takes
// the warp-wide max key and the lowest id holding it, then clears that key;
// k rounds, one redux pair each.
// SIG false: key = the logit, w = softmax over the k chosen logits.
// SIG true: s_e = sigmoid(l_e) in FP32, key = s_e + bias[e] (bias may be
// null), w = s_j / sum of the k chosen s.
// SMEM: the logits are in shared memory (else global memory, read through L2).
template <int PER, bool SMEM = false, bool SIG = false>  // logits per lane: E <= 32 * PER
__device__ __forceinline__ void warp_topk(const float *lg, int E, int k, int lane, int &id,
                                          float &w, const float *bias = nullptr) {
    uint32_t key[PER];
    float sv[PER];
#pragma unroll
    for (int m = 0; m < PER; ++m) {
        const int e = lane + 32 * m;
        const float l = e < E ? (SMEM ? lg[e] : __ldcg(lg + e)) : 0.f;
        if (SIG) {
            sv[m] = 1.0f / (1.0f + expf(-l));
            key[m] = e < E ? logit_key(sv[m] + (bias ? __ldg(bias + e) : 0.f)) : 0u;
        } else {
            key[m] = e < E ? logit_key(l) : 0u;
        }
    }
    id = -1;
    float mylv = 0.f, top = 0.f;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int bi = 0x7FFFFFFF;
#pragma unroll
        for (int m = 0; m < PER; ++m)
            if (key[m] > bk) {
                bk = key[m];
                bi = lane + 32 * m;
            }
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const int wi = (int)__reduce_min_sync(0xffffffffu, bk == wk ? (uint32_t)bi : 0x7FFFFFFFu);
        float lv = __uint_as_float((wk & 0x80000000u) ? (wk & 0x7FFFFFFFu) : ~wk);
        if (SIG) {
            // the chosen expert's unbiased score, from the lane that holds it
            float mine_s = 0.f;
#pragma unroll
            for (int m = 0; m < PER; ++m)
                if ((wi >> 5) == m) mine_s = sv[m];
            lv = __shfl_sync(0xffffffffu, mine_s, wi & 31);
        }
        if (j == 0) top = lv;
        if (lane == j) {
            id = wi;
            mylv = lv;
        }
#pragma unroll
        for (int m = 0; m < PER; ++m)
            if (wi == lane + 32 * m) key[m] = 0u;
    }
    // SIG: lane j < k holds s_j; else exp(l_j - l_0) (softmax)
    const float mine = lane < k ? (SIG ? mylv : expf(mylv - top)) : 0.f;
    float z = mine;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    w = mine / z;
}

// Larger expert counts: out of line, to keep the hot kernels' code small.
// Returns {id, w bits} (by value: no local-memory outputs).
template <bool SMEM, bool SIG = false>
static __device__ __noinline__ uint2 warp_topk_wide(const float *lg, int E, int k, int lane,
                                                    const float *bias) {
    int id;
    float w;
    warp_topk<32, SMEM, SIG>(lg, E, k, lane, id, w, bias);
    return make_uint2((unsigned)id, __float_as_uint(w));
}

// Dispatch on E (up to 1024 experts).
template <bool SMEM = false, bool SIG = false>
__device__ __forceinline__ void warp_topk_any(const float *lg, int E, int k, int lane, int &id,
                                              float &w, const float *bias = nullptr) {
    if (E <= 64)
        warp_topk<2, SMEM, SIG>(lg, E, k, lane, id, w, bias);
    else {
        const uint2 r = warp_topk_wide<SMEM, SIG>(lg, E, k, lane, bias);
        id = (int)r.x;
        w = __uint_as_float(r.y);
    }
}

// ------------------------------------------------------- gpu-scope words --
// Relaxed gpu-scope accesses (through L2, coherent across SMs).

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_gpu(unsigned *p, unsigned v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// {a, b} as one 64-bit scalar access (a in the low word): naturally aligned,
// it is single-copy atomic, so a reader sees both halves of one write.
__device__ __forceinline__ void st_relaxed_gpu_v2(uint2 *p, unsigned a, unsigned b) {
    asm volatile("{ .reg .b64 t; mov.b64 t, {%1, %2}; st.relaxed.gpu.global.b64 [%0], t; }" ::"l"(p),
                 "r"(a), "r"(b)
                 : "memory");
}
// Two such 64-bit words (each single-copy atomic on its own).
__device__ __forceinline__ void ld_relaxed_gpu_2x64(const uint2 *p, uint2 &a, uint2 &b) {
    asm volatile(
        "{ .reg .b64 t0, t1; ld.relaxed.gpu.global.v2.b64 {t0, t1}, [%4];"
        " mov.b64 {%0, %1}, t0; mov.b64 {%2, %3}, t1; }"
        : "=r"(a.x), "=r"(a.y), "=r"(b.x), "=r"(b.y)
        : "l"(p)
        : "memory");
}
__device__ __forceinline__ uint2 ld_relaxed_gpu_v2(const uint2 *p) {
    uint2 v;
    asm volatile("{ .reg .b64 t; ld.relaxed.gpu.global.b64 t, [%2]; mov.b64 {%0, %1}, t; }"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p)
                 : "memory");
    return v;
}

// ------------------------------------------- programmatic launch ---------

__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace moe
