// gemv.cuh — device building blocks shared by the decode kernels: in-kernel
// top-k into shared memory, the lane-team tools of the packed GEMV (chunk
// loads, FP16 activation staging, the E2M1 x FP16 chunk dot), the L2
// prefetch of the down matrices, the bulk-copy ring geometry, and the
// host-side launch helper (programmatic stream serialization).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "kernels.cuh"

namespace moe {

constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kDownWarps = kDownThreads / 32;

// One token's top-k by the calling warp into shared memory (ids) and,
// optionally, global memory (ids_out, w_out).  Out of line.
static __device__ __noinline__ void topk_token_to_smem(const float *lg, int E, int k, int *s_ids,
                                                int32_t *ids_out, float *w_out) {
    const int lane = threadIdx.x & 31;
    int id;
    float w;
    warp_topk_any(lg, E, k, lane, id, w);
    if (lane < k) {
        s_ids[lane] = id;
        if (ids_out) ids_out[lane] = id;
        if (w_out) w_out[lane] = w;
    }
}

// Routing inside the expert kernels: warp t of the CTA selects for token t
// (T <= kDecodeMaxT) into shared memory; CTA 0 also publishes ids / w.
// Out of line (runs once per call).
static __device__ __noinline__ void route_into_smem(const float *logits, int T, int E, int k,
                                                int *s_ids, float *s_w, int32_t *ids_out,
                                                float *w_out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp < T) {
        int id;
        float w;
        warp_topk_any(logits + (size_t)warp * E, E, k, lane, id, w);
        if (lane < k) {
            s_ids[warp * k + lane] = id;
            if (s_w) s_w[warp * k + lane] = w;
            if (blockIdx.x == 0 && ids_out) ids_out[warp * k + lane] = id;
            if (blockIdx.x == 0 && w_out) w_out[warp * k + lane] = w;
        }
    }
}

// ------------------------------------------------------------- team tools --
// A "team" of TL lanes (TL a power of two, aligned in the warp) owns one packed
// row at a time; lane lt of the team holds the KCH 16-byte chunks
// c = lt + TL*u (u < KCH) of the row (one E8M0 group each) and the matching
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
        const int c = lt + TL * u;
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

// NV: two E4M3 scale bytes per chunk (else one E8M0 byte); an absent chunk
// gets codes 0 and a unit scale.
template <int TL, int KCH, bool NV = false>
__device__ __forceinline__ void load_chunks(const uint8_t *codes, const uint8_t *scales, bool ok,
                                            int lt, int C, uint4 (&cw)[KCH], uint32_t (&sc)[KCH]) {
#pragma unroll
    for (int u = 0; u < KCH; ++u) {
        const int c = lt + TL * u;
        if (ok && c < C) {
            cw[u] = ld_stream16(codes + (size_t)c * 16);
            sc[u] = NV ? (ld_stream_u8(scales + 2 * c) | (ld_stream_u8(scales + 2 * c + 1) << 8))
                       : ld_stream_u8(scales + c);
        } else {
            cw[u] = make_uint4(0u, 0u, 0u, 0u);
            sc[u] = NV ? 0x3838u : 127u;
        }
    }
}

// NVFP4: each chunk's two 16-element half sums times their E4M3 scales.
template <int KCH>
__device__ __forceinline__ float chunks_dot_nv(const uint4 (&cw)[KCH], const uint32_t (&sc)[KCH],
                                               const uint32_t (&xw)[KCH][16]) {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < KCH; ++u) {
        float lo, hi, slo, shi;
        dot32_e2m1_f16_halves(cw[u], xw[u], lo, hi);
        e4m3x2_to_f32(sc[u], slo, shi);
        acc = fmaf(lo, slo, acc);
        acc = fmaf(hi, shi, acc);
    }
    return acc;
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
__device__ __forceinline__ void prefetch_down_slice(const GateUpParams &p, const int *s_ids,
                                                    int lane) {
    const int P = p.T * p.k;
    const int Pr = (P + 31) & ~31;  // every lane iterates the same number of times
    #pragma unroll 1
    for (int q = lane; q < Pr; q += 32) {
        const int e = q < P ? s_ids[q] : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const bool leader = (__ffs(same) - 1) == lane;
        if (q < P && leader && e >= 0 && e < p.E) {
            const size_t mc = (size_t)p.H * p.I / 2, ms = (size_t)p.H * p.I / 32;
            const size_t oc = (size_t)blockIdx.x * p.pf_codes;
            const size_t os = (size_t)blockIdx.x * p.pf_scales;
            const uint8_t *dc = p.codes_base ? p.codes_base + (size_t)(3 * e + 2) * p.codes_stride
                                             : p.table[e].codes[2];
            const uint8_t *ds = p.codes_base ? p.scales_base + (size_t)(3 * e + 2) * p.scales_stride
                                             : p.table[e].scales[2];
            if (oc < mc) {
                const size_t n = min((size_t)p.pf_codes, mc - oc);
                prefetch_l2_bulk(dc + oc, (uint32_t)n);
            }
            if (os < ms) {
                const size_t n = min((size_t)p.pf_scales, ms - os);
                prefetch_l2_bulk(ds + os, (uint32_t)n);
            }
        }
    }
}

// ------------------------------------------------- bulk-copy ring geometry --

constexpr int kTmaConsumers = 23;
constexpr int kTmaThreads = (kTmaConsumers + 1) * 32;
constexpr int kTmaSlotRows = kTmaConsumers;
constexpr int kTmaMaxSlots = 16;
constexpr size_t kTmaSmemBudget = 200 * 1024;

// nv: NVFP4 rows (an E4M3 scale per 16 elements instead of an E8M0 per 32).
__host__ __device__ __forceinline__ size_t tma_slot_bytes(int H, int nv = 0) {
    return (size_t)kTmaSlotRows * 2 * ((size_t)H / 2 + (size_t)H / (nv ? 16 : 32));
}

// ------------------------------------------------- gate / up ring phases --
// One CTA's share [cb, ce) of the gate/up items (rows of the selected
// experts' gate and up matrices, (pair, row) order) moves through a ring of
// shared-memory slots: slot s holds kTmaSlotRows consecutive items (gate
// codes, up codes, gate scales, up scales).  A producer warp issues bulk
// copies that complete on per-slot mbarriers; the consumer warps each take one
// row per slot.  Every wait is bounded; a timeout sets a status bit and the
// producer drains its outstanding copies before returning.

struct RingGeom {
    int cb, ce;          // items of this CTA
    int nsteps, nbar;    // slots to process, mbarrier pairs in use
    int nslots;
    size_t rc, rs;       // bytes of one row's codes / scales
    size_t slot_bytes, up_off, gs_off, us_off;
};

__device__ __forceinline__ RingGeom ring_geom(const GateUpParams &p) {
    RingGeom g;
    // this CTA's items [cb, ce): 32-bit math (T * k * I <= 4 * 8 * 4096), the
    // quotient computed in floating point and corrected
    const int N = p.T * p.k * p.I;
    const int G = (int)gridDim.x;
    auto split = [&](int c) {
        int v = (int)(((double)N * c) / G);
        while ((long long)v * G > (long long)N * c) --v;
        while ((long long)(v + 1) * G <= (long long)N * c) ++v;
        return v;
    };
    g.cb = split((int)blockIdx.x);
    g.ce = split((int)blockIdx.x + 1);
    g.nslots = p.nslots;
    g.nsteps = (g.ce - g.cb + kTmaSlotRows - 1) / kTmaSlotRows;
    g.nbar = min(g.nslots, g.nsteps);
    g.rc = (size_t)p.H >> 1;
    g.rs = (size_t)p.H >> (p.nv ? 4 : 5);
    g.slot_bytes = tma_slot_bytes(p.H, p.nv);
    g.up_off = (size_t)kTmaSlotRows * g.rc;
    g.gs_off = 2 * g.up_off;
    g.us_off = g.gs_off + (size_t)kTmaSlotRows * g.rs;
    return g;
}

// By one thread, before the CTA's first barrier.
__device__ __forceinline__ void ring_init(const RingGeom &g, uint64_t *full, uint64_t *empty) {
    #pragma unroll 1
    for (int s = 0; s < g.nbar; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], kTmaConsumers);
    }
    mbar_fence_init();
}

// Producer warp, once s_ids holds the call's routing: expert addresses, the
// ring fill, after_fill() (with the first copies in flight), the refills, the
// L2 prefetch of the down matrices, and the drain of every copy still in
// flight.
template <class AfterFill>
__device__ __forceinline__ void ring_produce(const GateUpParams &p, const RingGeom &g,
                                             uint8_t *ring, uint64_t *full, uint64_t *empty,
                                             const int *s_ids, ExpertPtrs *s_tab, int lane,
                                             AfterFill &&after_fill) {
    const int E = p.E, I = p.I;
    const int P = p.T * p.k;
    const int cb = g.cb, ce = g.ce, nsteps = g.nsteps, nbar = g.nbar, nslots = g.nslots;
    const size_t rc = g.rc, rs = g.rs, slot_bytes = g.slot_bytes;
    const size_t up_off = g.up_off, gs_off = g.gs_off, us_off = g.us_off;
    const uint64_t pol = l2_evict_first_policy();  // the rows are read once
    #pragma unroll 1
    for (int q = lane; q < P; q += 32) {
        const int e = s_ids[q];
        if (e >= 0 && e < E) {
            if (p.codes_base) {
                ExpertPtrs ep;
#pragma unroll
                for (int m = 0; m < 3; ++m) {
                    ep.codes[m] = p.codes_base + (size_t)(3 * e + m) * p.codes_stride;
                    ep.scales[m] = p.scales_base + (size_t)(3 * e + m) * p.scales_stride;
                }
                s_tab[q] = ep;
            } else {
                s_tab[q] = p.table[e];
            }
        }
    }
    __syncwarp();
    // Initial fill of the ring: one lane per (slot, pair segment, matrix)
    // copy, all in one round; lane 8 s + 0 also announces slot s's bytes.
    // Later slots reuse ring buffers and are issued by lane 0 in order.
    const int nfill = min(nsteps, nslots);
    #pragma unroll 1
    for (int task = lane; task < 8 * nfill; task += 32) {
        const int s = task >> 3, sub = task & 7, seg = sub >> 2, m = sub & 3;
        const int r0 = cb + s * kTmaSlotRows;
        const int r1 = min(ce, r0 + kTmaSlotRows);
        const int qa = r0 / I, qb = (r1 - 1) / I;  // at most two pairs per slot
        uint8_t *base = ring + (size_t)s * slot_bytes;
        if (sub == 0) {
            unsigned bytes = 0;
            #pragma unroll 1
            for (int q = qa; q <= qb; ++q) {
                const int e = s_ids[q];
                const int n = min(r1, (q + 1) * I) - max(r0, q * I);
                if (e >= 0 && e < E) bytes += (unsigned)(2 * n) * (unsigned)(rc + rs);
            }
            mbar_arrive_expect_tx(&full[s], bytes);
        }
        const int q = qa + seg;
        if (q <= qb) {
            const int e = s_ids[q];
            const int a = max(r0, q * I);
            const int n = min(r1, (q + 1) * I) - a;
            if (e >= 0 && e < E) {
                const size_t idx = (size_t)(a - r0), i0 = (size_t)(a - q * I);
                const ExpertPtrs &ep = s_tab[q];
                const size_t dst = m == 0   ? idx * rc
                                   : m == 1 ? up_off + idx * rc
                                   : m == 2 ? gs_off + idx * rs
                                            : us_off + idx * rs;
                const uint8_t *src = m == 0   ? ep.codes[0] + i0 * rc
                                     : m == 1 ? ep.codes[1] + i0 * rc
                                     : m == 2 ? ep.scales[0] + i0 * rs
                                              : ep.scales[1] + i0 * rs;
                const unsigned nb = (unsigned)(m < 2 ? n * rc : n * rs);
                bulk_g2s_hint(base + dst, src, nb, &full[s], pol);
            }
        }
    }
    __syncwarp();
    after_fill();
    bool ok = true;
    #pragma unroll 1
    for (int s = nfill; s < nsteps && ok && lane == 0; ++s) {
        const int b = s % nslots;
        if (!mbar_wait(&empty[b], (unsigned)((s / nslots) - 1) & 1u)) {
            atomicOr(p.status, kTimeoutStatus);
            ok = false;
            break;
        }
        uint8_t *base = ring + (size_t)b * slot_bytes;
        const int r0 = cb + s * kTmaSlotRows;
        const int r1 = min(ce, r0 + kTmaSlotRows);
        const int qa = r0 / I, qb = (r1 - 1) / I;
        unsigned bytes = 0;
        #pragma unroll 1
        for (int q = qa; q <= qb; ++q) {
            const int e = s_ids[q];
            const int n = min(r1, (q + 1) * I) - max(r0, q * I);
            if (e >= 0 && e < E) bytes += (unsigned)(2 * n) * (unsigned)(rc + rs);
        }
        mbar_arrive_expect_tx(&full[b], bytes);
        #pragma unroll 1
        for (int q = qa; q <= qb; ++q) {
            const int e = s_ids[q];
            const int a = max(r0, q * I);
            const int n = min(r1, (q + 1) * I) - a;
            if (e >= 0 && e < E) {
                const size_t idx = (size_t)(a - r0), i0 = (size_t)(a - q * I);
                const ExpertPtrs &ep = s_tab[q];
                bulk_g2s_hint(base + idx * rc, ep.codes[0] + i0 * rc, (unsigned)(n * rc),
                              &full[b], pol);
                bulk_g2s_hint(base + up_off + idx * rc, ep.codes[1] + i0 * rc,
                              (unsigned)(n * rc), &full[b], pol);
                bulk_g2s_hint(base + gs_off + idx * rs, ep.scales[0] + i0 * rs,
                              (unsigned)(n * rs), &full[b], pol);
                bulk_g2s_hint(base + us_off + idx * rs, ep.scales[1] + i0 * rs,
                              (unsigned)(n * rs), &full[b], pol);
            }
        }
    }
    __syncwarp();
    if (p.prefetch_down) prefetch_down_slice(p, s_ids, lane);
    // no copy may still be in flight into this CTA's shared memory at exit
    for (int s = max(0, nsteps - nbar) + lane; s < nsteps; s += 32)
        mbar_wait(&full[s % nslots], (unsigned)(s / nslots) & 1u);
}

// Consumer warps: one row per slot each.  get_x(tok, xw) fills the warp's
// FP16-staged activations of token tok and returns their scale 2^c;
// emit_h(index, bf16) stores h[q][i] (index q I + i).
template <int KCH, bool NV = false, class GetX, class EmitH>
__device__ __forceinline__ void ring_consume(const GateUpParams &p, const RingGeom &g,
                                             const uint8_t *ring, uint64_t *full,
                                             uint64_t *empty, const int *s_ids, int warp,
                                             int lane, GetX &&get_x, EmitH &&emit_h) {
    const int E = p.E, I = p.I, k = p.k;
    const int C = p.H >> 5;
    const int cb = g.cb, ce = g.ce, nsteps = g.nsteps, nslots = g.nslots;
    const size_t rc = g.rc, rs = g.rs, slot_bytes = g.slot_bytes;
    const size_t up_off = g.up_off, gs_off = g.gs_off, us_off = g.us_off;
    uint32_t xw[KCH][16];
    int cur_tok = -1;
    float xs = 1.f;
    bool failed = false;
    #pragma unroll 1
    for (int s = 0; s < nsteps; ++s) {
        const int b = s % nslots;
        const int row = cb + s * kTmaSlotRows + warp;
        if (row < ce && !failed) {
            // activations first: staging overlaps the slot's copies in flight
            const int tok = (row / I) / k;
            if (tok != cur_tok) {
                xs = get_x(tok, xw);
                cur_tok = tok;
            }
            if (!mbar_wait(&full[b], (unsigned)(s / nslots) & 1u)) {
                failed = true;
                if (lane == 0) atomicOr(p.status, kTimeoutStatus);
            } else {
                const int q = row / I;
                const int i = row - q * I;
                const int e = s_ids[q];
                const bool bad = e < 0 || e >= E;
                const uint8_t *base = ring + (size_t)b * slot_bytes;
                uint4 cg[KCH], cu[KCH];
                uint32_t sg[KCH], su[KCH];
#pragma unroll
                for (int u = 0; u < KCH; ++u) {
                    const int c = lane + 32 * u;
                    if (c < C && !bad) {
                        cg[u] = *reinterpret_cast<const uint4 *>(base + (size_t)warp * rc + (size_t)c * 16);
                        cu[u] = *reinterpret_cast<const uint4 *>(base + up_off + (size_t)warp * rc +
                                                                (size_t)c * 16);
                        if (NV) {
                            sg[u] = *reinterpret_cast<const uint16_t *>(base + gs_off + (size_t)warp * rs + 2 * c);
                            su[u] = *reinterpret_cast<const uint16_t *>(base + us_off + (size_t)warp * rs + 2 * c);
                        } else {
                            sg[u] = base[gs_off + (size_t)warp * rs + c];
                            su[u] = base[us_off + (size_t)warp * rs + c];
                        }
                    } else {
                        cg[u] = cu[u] = make_uint4(0u, 0u, 0u, 0u);
                        sg[u] = su[u] = NV ? 0x3838u : 127u;
                    }
                }
                float ag = NV ? chunks_dot_nv<KCH>(cg, sg, xw) : chunks_dot<KCH>(cg, sg, xw);
                float au = NV ? chunks_dot_nv<KCH>(cu, su, xw) : chunks_dot<KCH>(cu, su, xw);
                ag = warp_sum(ag);
                au = warp_sum(au);
                if (lane == 0) {
                    uint16_t out = 0;
                    if (!bad) {
                        // NVFP4: the expert's gate/up multiplier, folded into
                        // the exact power-of-two staging scale
                        const float sx = NV ? xs * __ldg(p.gscale + 2 * e) : xs;
                        const float g = round_bf16(ag * sx);
                        const float uu = round_bf16(au * sx);
                        const float sl = round_bf16(g / (1.0f + expf(-g)));
                        out = f32_to_bf16(sl * uu);
                    } else {
                        atomicOr(p.status, kBadExpertId);
                    }
                    emit_h((size_t)q * I + i, out);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[b]);
    }
}

// (TL, KCH) for K/32 = C chunks per row: a team of TL lanes, KCH chunks per lane.
inline void pick_team(int C, int &TL, int &KCH) {
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


// Launch with cudaLaunchKernelEx; `pdl` sets programmatic stream serialization
// so the kernel may start while the previous one drains.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
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

}  // namespace moe
