// down.cuh — device building blocks of the down GEMV + combine, shared by the
// standalone down kernel (decode.cu) and the one-launch layer kernel
// (layer.cu): the CTA's down rows copied into shared memory, the FP16 staging
// of the SwiGLU vectors h, the team loop over the CTA's output rows, and the
// sequential BF16 routing-weighted combine.
//
// Sources (model card "LFM2.5-24B-A2B — Packed MXFP4 Inference"): "Grouped
// top-4 expert execution" (grouped down GEMV; fused combine that keeps
// sequential BF16 multiply/add rounding) and table "Model and quantization".
#pragma once

#include "gemv.cuh"

namespace moe {

// Where expert e's down matrix lives: base + (3 e + 2) * stride when the
// weights were bound contiguously, else the device table.
struct DownSrc {
    const ExpertPtrs *table;
    const uint8_t *codes_base, *scales_base;
    size_t codes_stride, scales_stride;
};
__device__ __forceinline__ const uint8_t *dsrc_codes(const DownSrc &s, int e) {
    return s.codes_base ? s.codes_base + (size_t)(3 * e + 2) * s.codes_stride : s.table[e].codes[2];
}
__device__ __forceinline__ const uint8_t *dsrc_scales(const DownSrc &s, int e) {
    return s.codes_base ? s.scales_base + (size_t)(3 * e + 2) * s.scales_stride
                        : s.table[e].scales[2];
}

// Staged h layout: the 4 16-byte pieces of 32-element chunk c sit in the
// order q ^ ((c >> 1) & 3), so that the lanes of a team, reading piece q of
// consecutive chunks, hit 8 distinct bank groups (conflict-free 16-byte loads).
__device__ __forceinline__ int h_piece(int c, int q) { return (c << 2) | (q ^ ((c >> 1) & 3)); }

// Shared-memory offset of the down rows (after the staged h and the expert
// outputs), 16-byte aligned for the bulk copies.
__host__ __device__ __forceinline__ size_t down_rows_offset(int T, int k, int I, int R) {
    return ((size_t)T * k * I * 2 + (size_t)k * R * 4 + 15) & ~(size_t)15;
}
// Dynamic shared memory of the down phase with rows in shared memory (nv:
// NVFP4 rows, an E4M3 scale per 16 elements).
__host__ __device__ __forceinline__ size_t down_rows_smem(int T, int k, int I, int R, int nv = 0) {
    return down_rows_offset(T, k, I, R) + (size_t)k * R * ((size_t)I / 2 + (size_t)I / (nv ? 16 : 32));
}

// By one thread: the CTA's down rows [r0, r1) of every slot into shared memory
// (one bulk copy per slot, token segment and codes / scales), completing on
// *bar; rows of an invalid expert id are not fetched.  Out of line.
static __device__ __noinline__ void issue_down_rows(const DownSrc src, int E, int H, int I, int k,
                                                    const int *s_ids, int r0, int r1, int R,
                                                    uint8_t *rows_c, uint8_t *rows_s,
                                                    uint64_t *bar, int nv = 0) {
    const size_t rc = (size_t)I >> 1, rs = (size_t)I >> (nv ? 4 : 5);
    const uint64_t pol = l2_evict_first_policy();  // the rows are read once
    unsigned bytes = 0;
    #pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1) mbar_arrive_expect_tx(bar, bytes);
        #pragma unroll 1
        for (int a = r0; a < r1;) {
            const int t = a / H;
            const int b = min(r1, (t + 1) * H);
            const size_t n0 = (size_t)(a - t * H), cnt = (size_t)(b - a);
            #pragma unroll 1
            for (int j = 0; j < k; ++j) {
                const int e = s_ids[t * k + j];
                if (e < 0 || e >= E) continue;
                if (pass == 0) {
                    bytes += (unsigned)(cnt * (rc + rs));
                } else {
                    const size_t li = (size_t)j * R + (size_t)(a - r0);
                    bulk_g2s_hint(rows_c + li * rc, dsrc_codes(src, e) + n0 * rc,
                                  (unsigned)(cnt * rc), bar, pol);
                    bulk_g2s_hint(rows_s + li * rs, dsrc_scales(src, e) + n0 * rs,
                                  (unsigned)(cnt * rs), bar, pol);
                }
            }
            a = b;
        }
    }
}

// Stage the P BF16 vectors h[q][0..I) into shared memory as FP16 words, each
// scaled by 2^-c_q (c_q from the vector's max |h|); s_xs[q] = 2^c_q.  One pass
// over h: every 16-byte piece is read once (raw into sh, in the swizzled
// piece order of h_piece) while its max |h|
// goes to s_max[q] (warp max, then a shared atomic max on the non-negative
// float bits); after one barrier each thread converts its own pieces in place.
// s_max[0..P) must be zero on entry.  h is read through L2 (written by other
// CTAs of an earlier kernel or of this one).  Out of line: it runs once per
// call and keeps the kernel's code small.
static __device__ __noinline__ void stage_h_block(const uint16_t *h, int P, int I, uint32_t *sh,
                                           float *s_xs, unsigned *s_max) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n4 = I >> 3;  // 16-byte pieces per vector
    const int total = P * n4;
    const uint4 *hv = reinterpret_cast<const uint4 *>(h);
    uint4 *sv = reinterpret_cast<uint4 *>(sh);
    // every lane of a warp runs the same trip count (warp-wide votes inside)
#pragma unroll 1
    for (int base = warp * 32; base < total; base += kDownThreads) {
        const int i = base + lane;
        const bool valid = i < total;
        float m = 0.f;
        int q = -1;
        if (valid) {
            const uint4 v = __ldcg(hv + i);  // through L2: h may come from this grid
            q = i / n4;
            const int pi = i - q * n4;  // 8-element piece of vector q
            sv[q * n4 + h_piece(pi >> 2, pi & 3)] = v;
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int r = 0; r < 4; ++r)
                m = fmaxf(m, fmaxf(fabsf(bf16_to_f32(w4[r] & 0xFFFFu)),
                                   fabsf(bf16_to_f32(w4[r] >> 16))));
        }
        if (__all_sync(0xffffffffu, q == __shfl_sync(0xffffffffu, q, 0))) {
            m = warp_max(m);
            if (lane == 0 && q >= 0) atomicMax(s_max + q, __float_as_uint(m));
        } else if (valid) {
            atomicMax(s_max + q, __float_as_uint(m));
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int i = threadIdx.x; i < total; i += kDownThreads) {
        const float sf = pow2_neg(f16_stage_exponent(__uint_as_float(s_max[i / n4])));
        const uint4 v = sv[i];
        uint4 o;
        o.x = f32x2_to_f16x2(bf16_to_f32(v.x & 0xFFFFu) * sf, bf16_to_f32(v.x >> 16) * sf);
        o.y = f32x2_to_f16x2(bf16_to_f32(v.y & 0xFFFFu) * sf, bf16_to_f32(v.y >> 16) * sf);
        o.z = f32x2_to_f16x2(bf16_to_f32(v.z & 0xFFFFu) * sf, bf16_to_f32(v.z >> 16) * sf);
        o.w = f32x2_to_f16x2(bf16_to_f32(v.w & 0xFFFFu) * sf, bf16_to_f32(v.w >> 16) * sf);
        sv[i] = o;
    }
    if (threadIdx.x < P) s_xs[threadIdx.x] = pow2(f16_stage_exponent(__uint_as_float(s_max[threadIdx.x])));
    __syncthreads();
}

// As stage_h_block, from tagged words h_tag[q][i] = {tag, BF16 h} written by
// the CTAs of this grid (8-byte words, each single-copy atomic): every
// 8-element piece is re-read (bounded, with back-off) until its 8 words carry
// `tag`.  Returns false on a timeout, the same value in every thread.
// s_max[0..P) must be zero on entry.  Out of line.
static __device__ __noinline__ bool stage_h_tagged(const uint2 *h_tag, int P, int I, unsigned tag,
                                                   uint32_t *sh, float *s_xs, unsigned *s_max) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n4 = I >> 3;  // 8-element pieces per vector
    const int total = P * n4;
    uint4 *sv = reinterpret_cast<uint4 *>(sh);
    bool ok = true;
#pragma unroll 1
    for (int base = warp * 32; base < total; base += kDownThreads) {
        const int i = base + lane;
        const bool valid = i < total;
        float m = 0.f;
        int q = -1;
        if (valid) {
            const uint2 *src = h_tag + (size_t)i * 8;
            uint2 w[8];
            bool got = false;
            #pragma unroll 1
            for (int s = 0; s < kMaxSpin && !got; ++s) {
#pragma unroll
                for (int u = 0; u < 4; ++u) ld_relaxed_gpu_2x64(src + 2 * u, w[2 * u], w[2 * u + 1]);
                got = true;
#pragma unroll
                for (int u = 0; u < 8; ++u) got = got && w[u].x == tag;
                if (!got) __nanosleep(64);
            }
            ok = ok && got;
            const uint4 v = make_uint4((w[0].y & 0xFFFFu) | (w[1].y << 16),
                                       (w[2].y & 0xFFFFu) | (w[3].y << 16),
                                       (w[4].y & 0xFFFFu) | (w[5].y << 16),
                                       (w[6].y & 0xFFFFu) | (w[7].y << 16));
            q = i / n4;
            const int pi = i - q * n4;
            sv[q * n4 + h_piece(pi >> 2, pi & 3)] = v;
#pragma unroll
            for (int u = 0; u < 8; ++u) m = fmaxf(m, fabsf(bf16_to_f32(w[u].y & 0xFFFFu)));
        }
        if (__all_sync(0xffffffffu, q == __shfl_sync(0xffffffffu, q, 0))) {
            m = warp_max(m);
            if (lane == 0 && q >= 0) atomicMax(s_max + q, __float_as_uint(m));
        } else if (valid) {
            atomicMax(s_max + q, __float_as_uint(m));
        }
    }
    ok = __syncthreads_and(ok) != 0;
#pragma unroll 1
    for (int i = threadIdx.x; i < total; i += kDownThreads) {
        const float sf = pow2_neg(f16_stage_exponent(__uint_as_float(s_max[i / n4])));
        const uint4 v = sv[i];
        uint4 o;
        o.x = f32x2_to_f16x2(bf16_to_f32(v.x & 0xFFFFu) * sf, bf16_to_f32(v.x >> 16) * sf);
        o.y = f32x2_to_f16x2(bf16_to_f32(v.y & 0xFFFFu) * sf, bf16_to_f32(v.y >> 16) * sf);
        o.z = f32x2_to_f16x2(bf16_to_f32(v.z & 0xFFFFu) * sf, bf16_to_f32(v.z >> 16) * sf);
        o.w = f32x2_to_f16x2(bf16_to_f32(v.w & 0xFFFFu) * sf, bf16_to_f32(v.w >> 16) * sf);
        sv[i] = o;
    }
    if (threadIdx.x < P) s_xs[threadIdx.x] = pow2(f16_stage_exponent(__uint_as_float(s_max[threadIdx.x])));
    __syncthreads();
    return ok;
}

// The CTA's output rows r in [r0, r1) (r = t H + n) of every slot j: warp w
// serves slot j = w % k; its TL-lane teams take rows r0 + ti, r0 + ti + tps,
// ... two at a time, with the next pair fetched while the current one is
// reduced.  Rows come from shared memory (SR: copied there by issue_down_rows)
// or are streamed from global memory.  The expert output BF16(o) of row r and
// slot j goes to so[j R + (r - r0)].
// NW: warps of the CTA that take part (all of them).
template <int TL, int KCH, bool SR, bool NV = false, int NW = kDownWarps>
struct DownRows {
    int H, I, k, E, C, R, r0, r1, tps, j, lt, rr;
    unsigned mask;
    bool worker;
    size_t rc, rs;
    DownSrc src;
    const int *s_ids;
    const uint8_t *rows_c, *rows_s;
    uint4 cw[2][KCH];
    uint32_t sc[2][KCH];
    bool bad[2];

    __device__ __forceinline__ DownRows(int H_, int I_, int k_, int E_, int R_, int r0_, int r1_,
                                        const DownSrc &src_, const int *s_ids_,
                                        const uint8_t *rows_c_, const uint8_t *rows_s_)
        : H(H_), I(I_), k(k_), E(E_), R(R_), r0(r0_), r1(r1_), src(src_), s_ids(s_ids_),
          rows_c(rows_c_), rows_s(rows_s_) {
        constexpr int TPW = 32 / TL;
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        C = I >> 5;
        rc = (size_t)I >> 1;
        rs = (size_t)I >> (NV ? 4 : 5);
        lt = lane & (TL - 1);
        mask = team_mask<TL>(lane);
        const int groups = NW / k;  // warps per slot
        j = warp % k;
        const int gi = warp / k;
        tps = groups * TPW;  // teams per slot
        worker = gi < groups;
        rr = r0 + gi * TPW + lane / TL;
        bad[0] = bad[1] = false;
    }

    __device__ __forceinline__ void fetch(int rbase) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = rbase + u * tps;
            const bool valid = worker && r < r1;
            const int t = valid ? r / H : 0;
            const int n = r - t * H;
            const int e = valid ? s_ids[t * k + j] : 0;
            bad[u] = valid && (e < 0 || e >= E);
            const bool ok = valid && !bad[u];
            if (SR) {
                const size_t li = (size_t)j * R + (size_t)(r - r0);
                const uint8_t *dc = rows_c + li * rc, *ds = rows_s + li * rs;
#pragma unroll
                for (int v = 0; v < KCH; ++v) {
                    const int c = lt + TL * v;
                    if (ok && c < C) {
                        cw[u][v] = *reinterpret_cast<const uint4 *>(dc + (size_t)c * 16);
                        sc[u][v] = NV ? *reinterpret_cast<const uint16_t *>(ds + 2 * c) : ds[c];
                    } else {
                        cw[u][v] = make_uint4(0u, 0u, 0u, 0u);
                        sc[u][v] = NV ? 0x3838u : 127u;
                    }
                }
            } else {
                const uint8_t *dc = nullptr, *ds = nullptr;
                if (ok) {
                    dc = dsrc_codes(src, e) + (size_t)n * rc;
                    ds = dsrc_scales(src, e) + (size_t)n * rs;
                }
                load_chunks<TL, KCH, NV>(dc, ds, ok, lt, C, cw[u], sc[u]);
            }
        }
    }

    // Rows in shared memory (SR): the same steps, each chunk's codes and scale
    // read at use (no fetch ahead: fewer live registers, same bits).
    __device__ __forceinline__ void run_smem(const uint32_t *sh, const float *s_xs, float *so,
                                             unsigned *status, const float *s_gs) {
        #pragma unroll 1
        while (worker && rr < r1) {
            const int t = rr / H;
            const uint32_t *xv = sh + (size_t)(t * k + j) * (I >> 1);
            const float xs = NV ? s_xs[t * k + j] * s_gs[t * k + j] : s_xs[t * k + j];
            const int rb = rr + tps;
            const bool second = rb < r1 && rb / H == t;
            const int e = s_ids[t * k + j];
            const bool bad = e < 0 || e >= E;
            const size_t l0 = (size_t)j * R + (size_t)(rr - r0), l1 = (size_t)j * R + (size_t)(rb - r0);
            const uint8_t *dc0 = rows_c + l0 * rc, *ds0 = rows_s + l0 * rs;
            const uint8_t *dc1 = rows_c + l1 * rc, *ds1 = rows_s + l1 * rs;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int u = 0; u < KCH; ++u) {
                const int c = lt + TL * u;
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
                    const uint4 w0 = *reinterpret_cast<const uint4 *>(dc0 + (size_t)c * 16);
                    if (NV) {
                        float lo, hi, slo, shi;
                        dot32_e2m1_f16_halves(w0, x, lo, hi);
                        e4m3x2_to_f32(*reinterpret_cast<const uint16_t *>(ds0 + 2 * c), slo, shi);
                        a0 = fmaf(hi, shi, fmaf(lo, slo, a0));
                        if (second) {
                            const uint4 w1 = *reinterpret_cast<const uint4 *>(dc1 + (size_t)c * 16);
                            dot32_e2m1_f16_halves(w1, x, lo, hi);
                            e4m3x2_to_f32(*reinterpret_cast<const uint16_t *>(ds1 + 2 * c), slo, shi);
                            a1 = fmaf(hi, shi, fmaf(lo, slo, a1));
                        }
                    } else {
                        a0 = fmaf(dot32_e2m1_f16(w0, x), e8m0_to_f32(ds0[c]), a0);
                        if (second)
                            a1 = fmaf(dot32_e2m1_f16(*reinterpret_cast<const uint4 *>(dc1 + (size_t)c * 16), x),
                                      e8m0_to_f32(ds1[c]), a1);
                    }
                }
            }
            a0 = team_add<TL>(a0, mask);
            a1 = team_add<TL>(a1, mask);
            if (lt == 0) {
                so[j * R + (rr - r0)] = bad ? 0.f : round_bf16(a0 * xs);
                if (second) so[j * R + (rb - r0)] = bad ? 0.f : round_bf16(a1 * xs);
                if (bad) atomicOr(status, kBadExpertId);
            }
            rr = second ? rr + 2 * tps : rr + tps;
        }
    }

    // The loop, from the rows fetched by fetch(rr) (streamed rows; rows in
    // shared memory go through run_smem, no fetch needed); h staged in sh /
    // s_xs.  NV: s_gs[q] is pair q's down multiplier (folded into the exact
    // power-of-two staging scale).
    __device__ __forceinline__ void run(const uint32_t *sh, const float *s_xs, float *so,
                                        unsigned *status, const float *s_gs = nullptr) {
        if constexpr (SR) {
            run_smem(sh, s_xs, so, status, s_gs);
            return;
        }
        #pragma unroll 1
        while (worker && rr < r1) {
            const int t = rr / H;
            const uint32_t *xv = sh + (size_t)(t * k + j) * (I >> 1);
            const float xs = NV ? s_xs[t * k + j] * s_gs[t * k + j] : s_xs[t * k + j];
            // both rows of a step belong to token t unless the second crosses
            // into the next token; then it is recomputed in the next step
            const int rb = rr + tps;
            const bool second = rb < r1 && rb / H == t;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int u = 0; u < KCH; ++u) {
                const int c = lt + TL * u;
                if (c < C) {
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
                        dot32_e2m1_f16_halves(cw[0][u], x, lo, hi);
                        e4m3x2_to_f32(sc[0][u], slo, shi);
                        a0 = fmaf(hi, shi, fmaf(lo, slo, a0));
                        dot32_e2m1_f16_halves(cw[1][u], x, lo, hi);
                        e4m3x2_to_f32(sc[1][u], slo, shi);
                        a1 = fmaf(hi, shi, fmaf(lo, slo, a1));
                    } else {
                        a0 = fmaf(dot32_e2m1_f16(cw[0][u], x), e8m0_to_f32(sc[0][u]), a0);
                        a1 = fmaf(dot32_e2m1_f16(cw[1][u], x), e8m0_to_f32(sc[1][u]), a1);
                    }
                }
            }
            a0 = team_add<TL>(a0, mask);
            a1 = team_add<TL>(a1, mask);
            const bool b0 = bad[0], b1 = bad[1];
            const int rnext = second ? rr + 2 * tps : rr + tps;
            if (rnext < r1) fetch(rnext);
            if (lt == 0) {
                so[j * R + (rr - r0)] = b0 ? 0.f : round_bf16(a0 * xs);
                if (b0) atomicOr(status, kBadExpertId);
                if (second) {
                    so[j * R + (rb - r0)] = b1 ? 0.f : round_bf16(a1 * xs);
                    if (b1) atomicOr(status, kBadExpertId);
                }
            }
            rr = rnext;
        }
    }
};

// Sequential BF16 combine of rows [r0, r1) in slot order (wb = BF16(w),
// p = BF16(o wb), y = BF16(y + p)), then the optional residual add; o_keep
// receives the expert outputs when given.  All threads of the CTA.
__device__ __forceinline__ void down_combine(int r0, int r1, int H, int k, int R, const float *so,
                                             const float *s_w, const uint16_t *residual,
                                             uint16_t *y_out, uint16_t *o_keep) {
    #pragma unroll 1
    for (int r = r0 + (int)threadIdx.x; r < r1; r += kDownThreads) {
        const int t = r / H, n = r - t * H;
        float y = 0.f;
        for (int jj = 0; jj < k; ++jj) {
            const float o = so[jj * R + (r - r0)];
            const float wb = round_bf16(s_w[t * k + jj]);
            y = round_bf16(y + round_bf16(o * wb));
            if (o_keep) o_keep[((size_t)t * k + jj) * H + n] = f32_to_bf16(o);
        }
        if (residual) y = round_bf16(bf16_to_f32(residual[r]) + y);
        y_out[r] = f32_to_bf16(y);
    }
}

}  // namespace moe
